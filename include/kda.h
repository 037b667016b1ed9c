/*
 * kda.h -- C ABI of libkda, the Kimi Delta Attention (KDA) operator on NVIDIA
 * B200 (sm_100a).
 *
 * The operator (per head, per sequence; pages on Kimi K3):
 *
 *   log a_t = -5 * sigmoid(g_t)                    per key channel
 *   S_t     = Diag(a_t) S_{t-1}
 *             + beta_t k_t (v_t - (Diag(a_t) S_{t-1})^T k_t)^T
 *   o_t     = S_t^T q_t
 *
 *   "Kimi K3 发布核实与 Moonshot AI 主干架构演变" (dllmharness report), §3,
 *   "KDA 为什么不同于 MLA": a per-head state matrix; the per-channel
 *   retention alpha decays the old state first, the write strength beta with
 *   the current key and value then corrects it, and the query reads the
 *   updated state; training uses a form that is recurrent across chunks and
 *   parallel within a chunk.  Same page, "K3 对 Kimi Linear 的进一步修改",
 *   bullet 1: log-decay is a scaled sigmoid bounded below by -5, which keeps
 *   the reciprocal scaling inside a 16-token tile within BF16 range.
 *   "Kimi K3 模型架构解析：KDA、AttnRes 与 Stable LatentMoE", §二.2:
 *   S_t = Update(S_{t-1}, k_t, v_t), o_t = Read(S_t, q_t); §二.3: 96 heads,
 *   128-dimensional state channels per head.
 *
 * Conventions shared by every entry point
 *   - All tensors are dense and row-major (last index contiguous) in the
 *     layouts given below; every pointer must be 16-byte aligned.
 *   - Pointers named "device" must point to device memory of the current
 *     device.  The library never allocates: the caller owns every buffer,
 *     including the workspace.
 *   - q, k, v, g, beta and o share one element type (kda_dtype).  States
 *     (h0, hT, S) are always fp32.
 *   - g is the raw gate; the library applies log a = -5 sigmoid(g) itself.
 *     beta is already the write strength in [0, 1].  No query scale is
 *     applied (o = S^T q exactly).
 *   - Argument errors are detected on the host before any launch: nothing is
 *     written and nothing is launched.  Work is asynchronous on `stream`
 *     (a cudaStream_t; NULL = the legacy default stream).  Errors found by a
 *     kernel (malformed cu_seqlens, a bounded wait that ran out) set a
 *     per-device status word that kda_stream_status() reports.
 *   - Support: KDA_BF16 with dk = dv = 128 runs the tcgen05 tensor-core
 *     path; KDA_BF16 with dk = dv in {16, 32, 64} and KDA_FP32 with
 *     dk = dv in {16, 32, 64, 128} run an fp32 CUDA-core path (the fp32 test
 *     mode).  Anything else returns KDA_ERR_UNSUPPORTED, and so does a
 *     tensor-core call with T_tot > 2^31 - 64 (tokens are signed 32-bit
 *     TMA coordinates there).
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
    KDA_ERR_INVALID_ARGUMENT = 1, /* null/misaligned pointer, bad size     */
    KDA_ERR_UNSUPPORTED = 2,      /* dtype, head size or length not supported */
    KDA_ERR_WORKSPACE = 3,        /* workspace missing or too small        */
    KDA_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed  */
    KDA_ERR_TIMEOUT = 5,          /* a kernel's bounded wait ran out       */
    KDA_ERR_BAD_SEQLENS = 6       /* a kernel found cu_seqlens malformed   */
} kda_status;

typedef enum {
    KDA_BF16 = 0,
    KDA_FP32 = 1
} kda_dtype;

/*
 * Bytes of device workspace kda_chunk_fwd needs for these sizes (0 when it
 * needs none).  Pure host function; never fails (returns 0 for sizes that
 * kda_chunk_fwd would reject).
 */
KDA_API size_t kda_chunk_fwd_workspace_size(int32_t N, int64_t T_tot, int32_t H,
                                    int32_t dk, int32_t dv, kda_dtype dt);

/*
 * Chunked prefill (16-token chunks: parallel inside a chunk, recurrent
 * across chunks) over N packed sequences.
 *
 *   q, k, g     device [T_tot, H, dk]      (dt)
 *   v           device [T_tot, H, dv]      (dt)
 *   beta        device [T_tot, H]          (dt)
 *   h0          device [N, H, dk, dv] fp32 initial states, or NULL (= 0)
 *   cu_seqlens  device int32 [N+1], cu[0] = 0, non-decreasing, cu[N] = T_tot;
 *               sequence n owns tokens [cu[n], cu[n+1]).  NULL means N
 *               sequences of T_tot / N tokens each (T_tot % N must be 0).
 *               Zero-length sequences are allowed (hT = h0).
 *   o           device [T_tot, H, dv]      (dt) output, o_t = S_t^T q_t
 *   hT          device [N, H, dk, dv] fp32 final states, or NULL (not
 *               written).  hT may alias h0 exactly (in-place carry).
 *   workspace   device scratch of kda_chunk_fwd_workspace_size() bytes
 *               (may be NULL when that is 0); 256-byte aligned.
 *
 * N * H must be below 2^31.
 * Returns KDA_OK once the work is enqueued on `stream`.  Malformed
 * cu_seqlens contents are found on the device: the affected sequences are
 * skipped and kda_stream_status() returns KDA_ERR_BAD_SEQLENS.
 */
KDA_API kda_status kda_chunk_fwd(const void *q, const void *k, const void *v,
                         const void *g, const void *beta, const float *h0,
                         const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                         int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                         void *o, float *hT, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * kda_chunk_fwd with the output gate fused into the output store:
 *
 *   o_t = (S_t^T q_t) * sigmoid(z_t)     elementwise over the dv channels
 *
 * Page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对 Kimi Linear 的
 * 进一步修改", bullet 2: the output gate is an input-dependent, full-rank
 * channel gate; reading: o * sigmoid(z) per value channel, no normalisation.
 *
 *   z   device [T_tot, H, dv] (dt), the raw gate projection; required when
 *       T_tot > 0 (KDA_ERR_INVALID_ARGUMENT otherwise), 16-byte aligned.
 *
 * Every other argument, the workspace and the status contract are those of
 * kda_chunk_fwd; hT is the ungated final state.  The gate is applied to the
 * fp32 output values in registers, before the single rounding to dt.
 */
KDA_API kda_status kda_chunk_fwd_gated(const void *q, const void *k, const void *v,
                                       const void *g, const void *beta, const float *h0,
                                       const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                                       int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                       const void *z, void *o, float *hT, void *workspace,
                                       size_t workspace_bytes, void *stream);

/*
 * One decode step for B sequences x H heads: one token each.  Same
 * recurrence as the prefill (one token of it); S is updated in place.
 *
 *   q, k, g     device [B, H, dk]     (dt)
 *   v           device [B, H, dv]     (dt)
 *   beta        device [B, H]         (dt)
 *   S           device [B, H, dk, dv] fp32, read and overwritten
 *   o           device [B, H, dv]     (dt) output, read from the updated S
 *
 * A single pass over S: every state element is read once and written once.
 * B * H must be below 2^31.  Returns KDA_OK once the work is enqueued on
 * `stream` (B = 0 enqueues nothing); argument errors as for kda_chunk_fwd.
 */
KDA_API kda_status kda_decode_step(const void *q, const void *k, const void *v,
                           const void *g, const void *beta, float *S,
                           void *o, int32_t B, int32_t H, int32_t dk,
                           int32_t dv, kda_dtype dt, void *stream);

/*
 * Gradient of the prefill for L = <dO, O> + <dhT, hT> (training; page "Kimi
 * K3 发布核实与 Moonshot AI 主干架构演变", §3 "KDA 为什么不同于 MLA", item 3:
 * the chunked form serves training).  Gate log a = -5 sigmoid(g).
 *
 *   q, k, v, g, beta, h0, cu_seqlens, N, T_tot, H, dk, dv, dt  as for
 *               kda_chunk_fwd (the forward's inputs; the forward's outputs
 *               are not needed: the state is recomputed)
 *   dO          device [T_tot, H, dv]  (dt)  gradient of o
 *   dhT         device [N, H, dk, dv] fp32   gradient of hT, or NULL (= 0)
 *   dq, dk, dg  device [T_tot, H, dk]  (dt)  outputs
 *   dv          device [T_tot, H, dv]  (dt)  output
 *   dbeta       device [T_tot, H]      (dt)  output
 *   dh0         device [N, H, dk, dv] fp32   output (gradient of the initial
 *               state, h0 given or not), or NULL (not written)
 *   workspace   kda_chunk_bwd_workspace_size() bytes, 256-byte aligned:
 *               the state at every 16-token chunk boundary of every (sequence,
 *               head), and 16 token states per (sequence, head)
 *
 * fp32 arithmetic on CUDA cores: one CTA per (sequence, head) sweeps the
 * sequence forward keeping chunk-boundary states, then walks the chunks in
 * reverse, recomputing each chunk's token states from its checkpoint and
 * applying the token-level chain rule.  dk = dv in {16, 32, 64, 128};
 * KDA_BF16 or KDA_FP32.  Argument and workspace errors are reported before any
 * launch; a malformed cu_seqlens is reported by kda_stream_status().
 */
KDA_API size_t kda_chunk_bwd_workspace_size(int32_t N, int64_t T_tot, int32_t H, int32_t dk,
                                            int32_t dv, kda_dtype dt);
KDA_API kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *g,
                                 const void *beta, const float *h0, const int32_t *cu_seqlens,
                                 int32_t N, int64_t T_tot, int32_t H, int32_t dk, int32_t dv,
                                 kda_dtype dt, const void *dO, const float *dhT, void *dq,
                                 void *dk_, void *dv_, void *dg, void *dbeta, float *dh0,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * The operator with the unbounded gate of Kimi Linear, the one K3 replaced
 * (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对 Kimi Linear
 * 的进一步修改", bullet 1):
 *
 *   log a_t = -softplus(g_t)            (instead of -5 sigmoid(g_t))
 *
 * Without the -5 bound a 16-token tile's cumulative decay can leave the BF16
 * and fp32 ranges, so this variant runs on the fp32 CUDA-core chunk kernel
 * with every decay factor formed as the exponential of a direct sum over the
 * tokens it spans (each factor in [0, 1]; g = +inf forgets exactly).
 * Arguments, layouts and status as for kda_chunk_fwd (no workspace); dt
 * KDA_BF16 or KDA_FP32, dk = dv in {16, 32, 64, 128}.
 */
KDA_API kda_status kda_chunk_fwd_softplus(const void *q, const void *k, const void *v,
                                          const void *g, const void *beta, const float *h0,
                                          const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                                          int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                          void *o, float *hT, void *stream);

/* kda_decode_step with the unbounded gate log a = -softplus(g) (see above). */
KDA_API kda_status kda_decode_step_softplus(const void *q, const void *k, const void *v,
                                            const void *g, const void *beta, float *S,
                                            void *o, int32_t B, int32_t H, int32_t dk,
                                            int32_t dv, kda_dtype dt, void *stream);

/*
 * The step just before the operator, fused into one memory-bound pass: the
 * operator's inputs q, k, v, beta from the raw projections of the layer.
 * Page "Kimi K3 模型架构解析：KDA、AttnRes 与 Stable LatentMoE", §二.3 (a
 * length-4 short convolution mixes neighbouring tokens); readings where the
 * page is silent: the convolution is causal and depthwise, it restarts at
 * every sequence start, no activation follows it, and q and k are then
 * L2-normalised per (token, head):
 *
 *   q_t = xq'_t / |xq'_t|,  k_t = xk'_t / |xk'_t|,  v_t = xv'_t,
 *   x'_t = sum_{j=0..3} w[:, :, j] * x_{t-j}   (tokens before the sequence
 *                                               start count as zero)
 *   beta_t = sigmoid(beta_raw_t)
 *
 * An all-zero convolved row of q or k stays zero.  The gate g is not touched
 * (kda_chunk_fwd applies log a = -5 sigmoid(g) itself).
 *
 *   xq, xk, xv  device [T_tot, H, d]  (dt)  raw projections
 *   wq, wk, wv  device [H, d, 4] fp32       filter taps (tap j: token t - j)
 *   beta_raw    device [T_tot, H]     (dt)
 *   cu_seqlens  as for kda_chunk_fwd (NULL: N sequences of T_tot / N)
 *   q, k, v     device [T_tot, H, d]  (dt)  outputs (may not alias the inputs)
 *   beta        device [T_tot, H]     (dt)  output
 *
 * d in {16, 32, 64, 128}; dt KDA_BF16 or KDA_FP32 (fp32 arithmetic, outputs
 * rounded to dt); H <= 65535.  Argument errors are reported before any
 * launch; a malformed cu_seqlens is reported by kda_stream_status() as
 * KDA_ERR_BAD_SEQLENS (every access stays inside the buffers).
 */
KDA_API kda_status kda_prologue(const void *xq, const void *xk, const void *xv,
                                const float *wq, const float *wk, const float *wv,
                                const void *beta_raw, const int32_t *cu_seqlens, int32_t N,
                                int64_t T_tot, int32_t H, int32_t d, kda_dtype dt, void *q,
                                void *k, void *v, void *beta, void *stream);

/*
 * kda_chunk_fwd without a caller-provided workspace, for callers that cannot
 * allocate device memory: a serving engine that has reserved nearly all of
 * the GPU's memory for its own caches, a plugin whose host owns the
 * allocator, or latency-sensitive code that must not call cudaMalloc because
 * it can synchronise the device.  The pages have no counterpart; this is a
 * convenience of the library.
 *
 * Arguments and results are those of kda_chunk_fwd (without workspace and
 * workspace_bytes).  The scratch the long-sequence path needs (see
 * kda_chunk_fwd_workspace_size) comes from a static device array of 16 MiB
 * that every GPU loading libkda holds until the process exits; the call
 * allocates nothing.  A problem that needs more scratch than that returns
 * KDA_ERR_WORKSPACE before anything is launched.  The first call on a device
 * looks up the array's device address; make that first call before any
 * stream capture.  All calls on a device share the array: calls that may
 * overlap on the GPU (different streams, no ordering between them) race on
 * it and must not be issued.  Every scratch value a call reads is written
 * earlier in the same call, so leftover contents from an earlier call do not
 * matter.
 */
KDA_API kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                         const void *g, const void *beta, const float *h0,
                                         const int32_t *cu_seqlens, int32_t N, int64_t T_tot,
                                         int32_t H, int32_t dk, int32_t dv, kda_dtype dt,
                                         void *o, float *hT, void *stream);

/*
 * Synchronises `stream`, then returns and clears the current device's
 * status word: KDA_OK, KDA_ERR_TIMEOUT, KDA_ERR_BAD_SEQLENS, or
 * KDA_ERR_CUDA if the synchronisation itself failed.  The word is per
 * device, not per stream: a bit may come from a kernel on another stream of
 * the same device.  It is read and cleared in one atomic exchange (a one-
 * thread kernel on `stream`), so no bit raised meanwhile is lost; it is then
 * reported by the next call.
 */
KDA_API kda_status kda_stream_status(void *stream);

/*
 * Diagnostic of the failure-reporting path, with no fault: launches one tiny
 * kernel on `stream` whose single thread waits, with the same bounded wait as
 * the prefill pipeline, on a barrier that nothing ever arrives on.  After
 * limit_cycles SM clock cycles (1 .. 2^32; about 0.5 ns each) the wait gives
 * up and sets KDA_ERR_TIMEOUT in the status word, as a stalled pipeline stage
 * would; kda_stream_status() then reports it and the context stays usable.
 * Returns KDA_ERR_INVALID_ARGUMENT for a limit outside that range.
 */
KDA_API kda_status kda_selftest_wait_timeout(uint64_t limit_cycles, void *stream);

/*
 * Diagnostic of the prefill pipeline's own failure path, with no fault: the
 * NEXT kda_chunk_fwd call that runs the tensor-core path (KDA_BF16,
 * dk = dv = 128) makes the scan of every CTA wait, at state step `step`
 * (32 tokens each), on a barrier that nothing ever arrives on, and bounds
 * every pipeline wait of that call by limit_cycles SM clock cycles.  The
 * wait gives up, the kernel sets KDA_ERR_TIMEOUT in the status word, every
 * role of the CTA leaves its loop, the CTA waits for its own copies, stores
 * and tensor-core products, frees its tensor memory and returns; nothing is
 * written outside o and hT.  The values of that call's outputs are then
 * undefined.  The setting is consumed by that one call (process-wide, not
 * per device or stream).  Returns KDA_ERR_INVALID_ARGUMENT for step < 0 or a
 * limit outside 1 .. 2^32.
 */
KDA_API kda_status kda_debug_stall_prefill(int32_t step, uint64_t limit_cycles);

/*
 * Diagnostic (test-only) record of the magnitudes the tensor-core prefill
 * forms inside one step, the evidence for the bf16 range claim of the bounded
 * gate (page "Kimi K3 发布核实与 Moonshot AI 主干架构演变", §3 "K3 对 Kimi
 * Linear 的进一步修改", bullet 1: reciprocal decay scaling inside a 16-token
 * tile stays within the BF16 range).  kda_debug_range_prefill(step) clears the
 * record and makes CTA 0 (the first (sequence, head) chain) of the NEXT
 * tensor-core kda_chunk_fwd call record its operands at state step `step`
 * (32 tokens): the scaled keys Kr = K e^{b-m}, queries Qr = Q e^{b-m} and
 * keys Kh = K e^{m-b} as the gate pass writes them (bf16), and Z = Kh^T T
 * before the delta rescale (fp32, from tensor memory).  The setting is
 * consumed by that one call.  Returns KDA_ERR_INVALID_ARGUMENT for step < 0.
 *
 * kda_debug_range_read(out, n) copies the record, n >= 24 floats, row by row
 * for Kr, Qr, Kh, Z: max |x|, min nonzero |x|, then the counts of subnormal,
 * zero, non-finite and all values (as floats).  Call it after the prefill
 * completed (e.g. after kda_stream_status).
 */
KDA_API kda_status kda_debug_range_prefill(int32_t step);
KDA_API kda_status kda_debug_range_read(float *out, size_t n);

/* Static English description of a status code (never NULL). */
KDA_API const char *kda_status_string(kda_status s);

/* Library ABI version: major * 10000 + minor * 100 + patch. */
KDA_API int32_t kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H */
