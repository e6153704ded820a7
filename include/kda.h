/*
 * kda.h -- C ABI of the B200 (sm_100a) KDA operator library, libkda_b200.so.
 *
 * KDA (Kimi Delta Attention) is the linear-attention recurrence of
 * "Hybrid Linear Attention Architectures: Breaking Through the Long-Context
 * Engineering Bottleneck in LLMs", section "Core Module Design", Stage 3:
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *     o_t = S_t^T q_t,      alpha_t = exp(log_alpha_t)  (per key channel)
 *
 * S is d_k x d_v (rows = key channels).  The write term is read as k v^T (the
 * printed "v k^T" cannot be left-multiplied by the d_k x d_k erase matrix);
 * the decay acts before the erase (section 2.5 of "Linear Attention KDA Gating
 * in a 3:1 Hybrid Architecture"); the output is read after the write; q is not
 * scaled.
 *
 * Entry points: KDA prefill (kda_chunk_fwd, its static-workspace form
 * kda_chunk_fwd_static_ws, and the token-by-token kda_recurrent_fwd) and decode
 * (kda_decode_step); the same from the raw projections (kda_chunk_fwd_fused,
 * kda_decode_step_fused); Gated DeltaNet and DeltaNet (gdn_chunk_fwd,
 * gdn_recurrent_fwd, gdn_decode_step); the gradient of the prefill
 * (kda_chunk_bwd); status helpers.
 *
 * Conventions for every call
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates no device memory and keeps no pointer after the call returns.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *    means the legacy default stream).  Arguments are validated on the host
 *    before anything is launched; a rejected call launches nothing.
 *  - Tensors are dense, row-major, with every pointer 16-byte aligned.
 *  - `dtype` is the element type of q, k, v, log_alpha and beta (or of the
 *    tensors in their places: log_g, the raw projections); `out_dtype`
 *    that of out (KDA_F32 keeps the full accuracy of the fp32 accumulators:
 *    rounding the output to bf16 alone moves it by up to 2^-8 of its
 *    magnitude).  Recurrent states are always fp32.
 *  - No call throws across the ABI or exits the process; every failure is a
 *    kda_status.  KDA_ERR_CUDA means a launch or runtime call failed (use
 *    cudaGetLastError for details).
 *  - Kernels bound every wait they perform.  A wait that runs out records
 *    KDA_ERR_TIMEOUT in a device-side error word and the kernel returns early
 *    (its outputs are then undefined); kda_get_last_device_error reads it.
 */
#ifndef KDA_B200_KDA_H
#define KDA_B200_KDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misaligned pointer, bad cu_seqlens size */
    KDA_ERR_UNSUPPORTED = 2,   /* valid but not implemented: head size, chunk size, dtype */
    KDA_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 4        /* a kernel gave up on a bounded wait (device error word) */
} kda_status;

typedef enum {
    KDA_F32 = 0,   /* float32 I/O */
    KDA_BF16 = 1   /* bfloat16 I/O (fp32 accumulation and fp32 state) */
} kda_dtype;

/*
 * kda_chunk_fwd -- chunkwise-parallel prefill.
 *
 * Computes, for every sequence and head, the outputs o_t of all tokens and the
 * state after the last token, using the chunkwise form of the recurrence
 * ("Hardware-Aware Chunkwise Parallelism" on the page named above: the
 * inter-chunk state update and the intra-chunk output equations; section 3 of
 * "Linear Attention KDA Gating in a 3:1 Hybrid Architecture").  Within a chunk
 * the per-channel log decays are summed, the WY factors W and U come from the
 * UT transform T = (I + strict_tril(diag(beta)(K*Gamma)(K/Gamma)^T))^{-1}, and
 *     U~ = U - W S,   O = (Q*Gamma) S + tril((Q*Gamma)(K/Gamma)^T) U~,
 *     S <- Diag(gamma) S + (K*gamma/Gamma)^T U~.
 * The result equals the token recurrence up to rounding.
 *
 *   q, k, log_alpha : [B, T, H, d_k]  dtype.  log_alpha <= 0 (alpha in (0, 1]).
 *   v               : [B, T, H, d_v]  dtype.
 *   beta            : [B, T, H]       dtype, in [0, 1].
 *   init_state      : [N, H, d_k, d_v] fp32, or NULL for zero initial states.
 *   cu_seqlens      : NULL, or int32 [num_seqs + 1] (device) with B == 1:
 *                     packed sequences, sequence n = tokens cu_seqlens[n] ..
 *                     cu_seqlens[n+1]-1; ascending, cu_seqlens[0] == 0,
 *                     cu_seqlens[num_seqs] == T (not checked on the host:
 *                     reading it would need a device sync).  Chunks never
 *                     cross sequences; empty sequences are allowed.
 *   N               : num_seqs when cu_seqlens is given, else B.
 *   chunk           : chunk length C, 1 <= C <= 64 (KDA_ERR_UNSUPPORTED above:
 *                     the tensor-core kernel's tiles are 64 tokens high, and a
 *                     chunk shorter than 64 fills their first C rows, like the
 *                     short last chunk of a sequence).  The result is the same
 *                     for every C up to rounding; C trades the length of the
 *                     sequential chain of chunk steps against the work per step.
 *   out             : [B, T, H, d_v] out_dtype (written).
 *   final_state     : [N, H, d_k, d_v] fp32, or NULL to skip.  It may alias
 *                     init_state exactly (in-place state update); partial
 *                     overlap is invalid.
 *   workspace       : device scratch of at least the size that
 *                     kda_chunk_fwd_workspace_size reports (16-byte aligned);
 *                     may be NULL when that size is 0.  Owned by the caller,
 *                     used only during the call; calls that overlap on the
 *                     GPU must not share one workspace.
 * Supported: d_k, d_v in {64, 128} for both dtypes.  bf16 runs on the tensor-
 * core path (with d_k == 64 the key channels are zero-padded to 128 inside the
 * kernel: the padded state rows stay zero and reach no output); fp32 I/O runs
 * token by token on CUDA cores with the fp32 state (fp32 accuracy; the chunk
 * length does not apply there).
 * T == 0 is valid (final_state = init_state or zeros).
 * The tensor-core path launches one CTA per SM of the device as a cooperative
 * grid (its CTAs wait on one another, so all must be resident at once); the
 * launch fails (KDA_ERR_CUDA) rather than start when the GPU cannot hold them
 * all, e.g. while another kernel occupies some SMs.
 */
kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *beta, const float *init_state, const int32_t *cu_seqlens,
                         int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t d_k,
                         int32_t d_v, int32_t chunk, kda_dtype dtype, kda_dtype out_dtype,
                         void *out, float *final_state, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * Workspace kda_chunk_fwd needs, in bytes, for N sequences (B, or num_seqs with
 * cu_seqlens) of H heads: on the tensor-core path, about 7 KB of schedule
 * tables (ring flags, sequence order) and, for each of up to min(N * H, 64)
 * chains, a ring of 12 chunk images (73 KB each at d_v = 128, 65 KB at
 * d_v = 64) through which the CTAs that prepare the chunk operands hand them
 * to the CTA that runs the state recurrence; 0 on the fp32 path.  Pure host
 * computation.  KDA_ERR_UNSUPPORTED (and *bytes = 0) for the shapes that
 * kda_chunk_fwd rejects with that status: d_k or d_v outside {64, 128}, and
 * KDA_BF16 with d_k != 128.
 */
kda_status kda_chunk_fwd_workspace_size(int32_t N, int32_t H, int32_t d_k, int32_t d_v,
                                        kda_dtype dtype, size_t *bytes);

/*
 * kda_recurrent_fwd -- the same operation as kda_chunk_fwd, evaluated token by
 * token on CUDA cores with the state in fp32 registers (the RNN mode that
 * section 3 of "Linear Attention KDA Gating in a 3:1 Hybrid Architecture"
 * contrasts with the chunked algorithm).  Same arguments and layouts as
 * kda_chunk_fwd without `chunk`; d_k, d_v in {64, 128}; either dtype.
 */
kda_status kda_recurrent_fwd(const void *q, const void *k, const void *v, const void *log_alpha,
                             const void *beta, const float *init_state,
                             const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                             int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                             kda_dtype out_dtype, void *out, float *final_state, void *stream);

/*
 * kda_decode_step -- one recurrent step for one new token per sequence, with
 * the fp32 state updated in place (the memory-bound decode step: every state
 * element is read once and written once).
 *
 *   q, k, log_alpha : [B, H, d_k] dtype;  v : [B, H, d_v] dtype;  beta : [B, H] dtype.
 *   state           : [B, H, d_k, d_v] fp32, read and overwritten.
 *   out             : [B, H, d_v] out_dtype (written).
 * Supported: d_k, d_v in {64, 128}.
 */
kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *log_alpha,
                           const void *beta, float *state, void *out, int32_t B, int32_t H,
                           int32_t d_k, int32_t d_v, kda_dtype dtype, kda_dtype out_dtype,
                           void *stream);

/*
 * Gated DeltaNet and DeltaNet -- the same recurrence with a coarser gate.  Gated
 * DeltaNet decays the whole state of a head by one factor per token,
 *     S_t = (I - beta_t k_t k_t^T) g_t S_{t-1} + beta_t k_t v_t^T,   g_t = exp(log_g_t),
 * the scalar-gate case of KDA: every key channel shares alpha_t = g_t, and a
 * scalar commutes with the erase, so g_t (I - beta k k^T) S equals
 * (I - beta k k^T) g_t S.  DeltaNet has no decay (g_t = 1).  Stages 1 and 2 of
 * section "Core Module Design" of "Hybrid Linear Attention Architectures:
 * Breaking Through the Long-Context Engineering Bottleneck in LLMs" define both.
 *
 * gdn_chunk_fwd, gdn_recurrent_fwd and gdn_decode_step take the same arguments,
 * layouts, paths, workspace (kda_chunk_fwd_workspace_size) and status codes as
 * kda_chunk_fwd, kda_recurrent_fwd and kda_decode_step, with log_g in place of
 * log_alpha:
 *   log_g : [B, T, H] dtype (prefill) or [B, H] dtype (decode), log_g <= 0, or
 *           NULL for DeltaNet (no decay; allowed whatever T is).
 */
kda_status gdn_chunk_fwd(const void *q, const void *k, const void *v, const void *log_g,
                         const void *beta, const float *init_state, const int32_t *cu_seqlens,
                         int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t d_k,
                         int32_t d_v, int32_t chunk, kda_dtype dtype, kda_dtype out_dtype,
                         void *out, float *final_state, void *workspace, size_t workspace_bytes,
                         void *stream);
kda_status gdn_recurrent_fwd(const void *q, const void *k, const void *v, const void *log_g,
                             const void *beta, const float *init_state,
                             const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                             int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                             kda_dtype out_dtype, void *out, float *final_state, void *stream);
kda_status gdn_decode_step(const void *q, const void *k, const void *v, const void *log_g,
                           const void *beta, float *state, void *out, int32_t B, int32_t H,
                           int32_t d_k, int32_t d_v, kda_dtype dtype, kda_dtype out_dtype,
                           void *stream);

/*
 * kda_chunk_fwd_fused / kda_decode_step_fused -- KDA from the raw projections,
 * with the step just before the recurrence done inside the kernels' loads
 * (the per-chunk gating parameters of the "Implementation checklist" of
 * "Hybrid Linear Attention Architectures: Breaking Through the Long-Context
 * Engineering Bottleneck in LLMs"), so that no separate pass writes the
 * normalised inputs to memory and reads them back:
 *     q = q_raw * rsqrt(sum(q_raw^2) + 1e-6),  k likewise   (L2 over d_k, per token and head)
 *     log_alpha = logsigmoid(g_raw),  beta = sigmoid(b_raw)
 * q_raw, k_raw, g_raw take the places (and layouts) of q, k, log_alpha and
 * b_raw that of beta; everything else is as in kda_chunk_fwd / kda_decode_step.
 * kda_chunk_fwd_fused runs on the tensor-core path only (dtype KDA_BF16;
 * KDA_ERR_UNSUPPORTED otherwise); kda_decode_step_fused supports what
 * kda_decode_step does.
 */
kda_status kda_chunk_fwd_fused(const void *q_raw, const void *k_raw, const void *v, const void *g_raw,
                               const void *b_raw, const float *init_state,
                               const int32_t *cu_seqlens, int32_t num_seqs, int32_t B, int32_t T,
                               int32_t H, int32_t d_k, int32_t d_v, int32_t chunk, kda_dtype dtype,
                               kda_dtype out_dtype, void *out, float *final_state, void *workspace,
                               size_t workspace_bytes, void *stream);
kda_status kda_decode_step_fused(const void *q_raw, const void *k_raw, const void *v,
                                 const void *g_raw, const void *b_raw, float *state, void *out,
                                 int32_t B, int32_t H, int32_t d_k, int32_t d_v, kda_dtype dtype,
                                 kda_dtype out_dtype, void *stream);

/*
 * kda_chunk_fwd_static_ws -- kda_chunk_fwd for callers that cannot allocate
 * device memory when they call it.  Examples: an inference engine that has
 * reserved all device memory up front in its own pool and forbids further
 * allocations, or code running inside an allocation callback, where calling
 * back into the allocator is not allowed.  Such a caller has no way to
 * provide the workspace argument of kda_chunk_fwd.  This call instead takes
 * the chunk-image handoff buffer from a fixed array built into the library
 * (KDA_STATIC_WS_BYTES per GPU; every GPU that loads the library holds it
 * until the process exits).  The pages describe nothing like it; it exists
 * only for such callers.
 *
 * Same arguments, layouts and results as kda_chunk_fwd, without workspace /
 * workspace_bytes.  Only the tensor-core path: dtype KDA_BF16, d_k in {64, 128},
 * d_v in {64, 128}.  It allocates nothing (no cudaMalloc, no library
 * allocator).  Any number of (sequence, head) pairs fits: the chains' rings
 * are made shallower (down to 3 images) when the array cannot hold 12 each.
 *
 * Each call looks up the current device's copy of the array (with that
 * device current) and caches its address per device; during stream capture
 * the cached address is used, so make the first call on a device before any
 * capture.  Outside capture the address is looked up again on every call, so
 * a device reset (cudaDeviceReset) between calls is harmless; a graph captured
 * before such a reset keeps the old address and must be captured again.
 * Every call on a device shares the one array and leaves its last contents
 * there; nothing in it needs to start at zero, since each chunk image is
 * written before it is read.  Two calls that run on the same GPU at the same
 * time (different streams, or graph replays in flight together) use the same
 * array and race: serialise them.
 */
#define KDA_STATIC_WS_BYTES (16u << 20)
kda_status kda_chunk_fwd_static_ws(const void *q, const void *k, const void *v, const void *log_alpha,
                                   const void *beta, const float *init_state,
                                   const int32_t *cu_seqlens, int32_t num_seqs, int32_t B,
                                   int32_t T, int32_t H, int32_t d_k, int32_t d_v, int32_t chunk,
                                   kda_dtype dtype, kda_dtype out_dtype, void *out,
                                   float *final_state, void *stream);

/*
 * kda_chunk_bwd -- gradient of kda_chunk_fwd with respect to every input
 * (reverse mode through the recurrence of "Core Module Design", Stage 3, of
 * the page named above; the pages train the layer -- the implementation
 * checklist there asks for FP32 intermediates and gradient clipping, and
 * section 3 of "Linear Attention KDA Gating in a 3:1 Hybrid Architecture"
 * asks for gradient checks -- but print no backward pass).  With w = S'^T k,
 * S' = Diag(alpha) S_prev and u = beta (v - w), one reverse token step is
 *     dS += q do^T;  dq = S do;  du = dS^T k;  dk = dS u - beta S' du;
 *     dbeta = du . (v - w);  dv = beta du;  dS' = dS - beta k du^T;
 *     dlog_alpha = rowsum(dS' * S');  dS_prev = Diag(alpha) dS'.
 * All arithmetic is fp32 on CUDA cores.  One cluster of d_v / 32 CTAs per
 * (sequence, head) keeps the state and its gradient in registers, each CTA a
 * 32-column slice; sums over d_k and d_v (the latter across the cluster through
 * distributed shared memory) run in a fixed order (results are reproducible
 * run to run).
 *
 *   q, k, v, log_alpha, beta, init_state, cu_seqlens, num_seqs, B, T, H,
 *   d_k, d_v, dtype : as for kda_chunk_fwd (the forward's inputs).
 *   chunk           : states are checkpointed every `chunk` tokens and each
 *                     chunk's per-token states recomputed from its checkpoint
 *                     (1 <= chunk <= 256); 0 keeps the state before every
 *                     token instead (no recompute: one pass fewer, a workspace
 *                     of H * total_tokens * d_k * d_v * 4 bytes).  It changes
 *                     no result: the gradients are bitwise the same.
 *   d_out           : [B, T, H, d_v] d_out_dtype, dLoss/dout.
 *   d_final_state   : [N, H, d_k, d_v] fp32 dLoss/dfinal_state, or NULL (zero).
 *   dq, dk, dlog_alpha : [B, T, H, d_k] fp32 (written).
 *   dv              : [B, T, H, d_v] fp32 (written).
 *   dbeta           : [B, T, H] fp32 (written).
 *   d_init_state    : [N, H, d_k, d_v] fp32 dLoss/dinit_state, or NULL to skip.
 *   workspace       : at least kda_chunk_bwd_workspace_size bytes (16-byte
 *                     aligned, owned by the caller): the checkpoints and one
 *                     chunk of per-token states for every (sequence, head).
 * Supported: d_k, d_v in {64, 128}; either dtype and d_out dtype.
 */
kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *log_alpha,
                         const void *beta, const float *init_state, const int32_t *cu_seqlens,
                         int32_t num_seqs, int32_t B, int32_t T, int32_t H, int32_t d_k,
                         int32_t d_v, int32_t chunk, kda_dtype dtype, const void *d_out,
                         kda_dtype d_out_dtype, const float *d_final_state, float *dq, float *dk,
                         float *dv, float *dlog_alpha, float *dbeta, float *d_init_state,
                         void *workspace, size_t workspace_bytes, void *stream);

/*
 * Workspace of kda_chunk_bwd, in bytes, for N sequences of H heads holding
 * total_tokens tokens in all (B * T, or the packed length with cu_seqlens).
 * Pure host computation; KDA_ERR_UNSUPPORTED for the shapes kda_chunk_bwd
 * rejects with that status.
 */
kda_status kda_chunk_bwd_workspace_size(int32_t N, int32_t H, int64_t total_tokens, int32_t d_k,
                                        int32_t d_v, int32_t chunk, size_t *bytes);

/* Human-readable name of a status (static string, never NULL). */
const char *kda_status_string(kda_status s);

/*
 * Synchronises `stream`, then returns and clears the device-side error word
 * of the current device: KDA_OK, or KDA_ERR_TIMEOUT if a kernel gave up on a
 * bounded wait since the last call.  KDA_ERR_CUDA if the sync or read failed.
 */
kda_status kda_get_last_device_error(void *stream);

/* Library version string, e.g. "kda_b200 0.2.0 sm_100a". */
const char *kda_version(void);

/*
 * Testing hook (not part of the operator): makes the tensor-core prefill's
 * failure path observable without a GPU fault.  After this call, every
 * launch of the prefill's tensor-core kernel (kda_chunk_fwd, gdn_chunk_fwd,
 * kda_chunk_fwd_fused, kda_chunk_fwd_static_ws) leaves the chunk image of
 * producer item `skip_item` unpublished (-1: none, the default), and every
 * wait on a ring flag gives up after `flag_wait_us` microseconds (0: the
 * default of 2 s).  A launch whose image is missing then ends on its own:
 * the waiting CTA records KDA_ERR_TIMEOUT in the device error word, raises
 * the launch's abort word, and every CTA leaves its loops and frees its
 * Tensor Memory; the outputs of that launch are undefined, and
 * kda_get_last_device_error reports KDA_ERR_TIMEOUT.  Items are numbered in
 * schedule order (item i is chunk i / C of chain i % C for C chains), so any
 * value below the number of chunks of the launch takes effect.  Process-wide;
 * not thread-safe against concurrent prefill calls.  KDA_ERR_INVALID_ARG for
 * skip_item < -1.
 */
kda_status kda_testing_set_chunk_fault(int32_t skip_item, uint32_t flag_wait_us);

#ifdef __cplusplus
}
#endif

#endif /* KDA_B200_KDA_H */
