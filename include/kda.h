/*
 * kda.h — C ABI of libkda, the B200 (sm_100a) implementation of the Kimi Delta Attention (KDA)
 * gated delta-rule recurrence.
 *
 * The recurrence, per (sequence, head), with state S in R^{d_k x d_v} (row = key channel,
 * column = value channel), for each token t:
 *   g_t   = -5 * sigmoid(exp(A_h) * a_t)          per-key-channel log-decay in [-5, 0]
 *   S     = Diag(exp(g_t)) S                      fade
 *   S     = S + beta_t k_t (v_t - S^T k_t)^T      erase what k_t retrieves, write v_t
 *   o_t   = S^T (scale * q_t)                     read (after the token's own write)
 *   out_t = sigmoid(gate_t) (.) o_t               full-rank output gate
 * Sources: "Review A · Sequence and depth", Free recall (fade, erase, write, then the read S^T q);
 * "Kimi K3 · Lesson 3 of 14" (chunkwise form, 16-token tiles, g_min = -5 scaled-sigmoid decay of
 * §2.1.1 eq. 5, full-rank output gate); "K3 Architecture Illustrated", §"Combining KDA and MLA",
 * FIG 21 (retention first, then the delta update, then the query read).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, densely packed
 *     (row-major, innermost dimension last).  Per-channel tensors (q, k, v, a, gate, out, states)
 *     must be 16-byte aligned; beta, A_log and cu_seqlens 4-byte aligned.  bf16 is IEEE bfloat16
 *     stored as uint16_t.  The caller owns every buffer; the library allocates nothing and keeps no state
 *     between calls except one per-device error word (see kda_sync_check).
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are asynchronous:
 *     a KDA_OK return means the work was validated and enqueued.
 *   - Argument errors are detected on the host before anything is enqueued and return
 *     KDA_ERR_INVALID_ARG or KDA_ERR_UNSUPPORTED.  A launch failure returns KDA_ERR_CUDA.
 *     Errors that can only be seen on the device (malformed cu_seqlens, a max_seqlen smaller
 *     than a sequence) are recorded in the per-device error word and reported by
 *     kda_sync_check; the affected outputs are then unspecified.  Kernels never trap.
 *   - Supported head sizes: d_k, d_v in {64, 128}.  g_min = -5, chunk = 64 tokens and
 *     tile = 16 tokens are compile-time constants.
 */
#ifndef KDA_H_
#define KDA_H_

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

typedef enum kda_status {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1, /* NULL required pointer, bad size, misaligned pointer, small workspace */
    KDA_ERR_UNSUPPORTED = 2, /* d_k or d_v outside {64, 128} */
    KDA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    KDA_ERR_TIMEOUT = 4,     /* a bounded device-side wait gave up (reported by kda_sync_check) */
    KDA_ERR_RANGE = 5        /* a prefill state ended non-finite: an fp16 tensor-core operand
                                (value, state, pseudo-value) left +-65504 (reported by kda_sync_check) */
} kda_status;

/* Storage type of the output o.  The recurrence itself is computed in fp32 either way. */
typedef enum kda_dtype {
    KDA_DTYPE_BF16 = 0,
    KDA_DTYPE_F32 = 1
} kda_dtype;

/*
 * kda_chunk_fwd — prefill over packed variable-length sequences, in the chunkwise form
 * ("Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram: O = (Gamma (.) Q) S + A V~, state carried
 * sequentially between 64-token chunks, every 16-token tile a dense product thanks to the
 * g_min = -5 bound).
 *
 * Layout: token-major, packed.  Sequence n owns tokens [cu_seqlens[n], cu_seqlens[n+1]).
 *   q, k, a     bf16  [total_tokens, H, d_k]   query, key, decay logits
 *   v           bf16  [total_tokens, H, d_v]
 *   beta        fp32  [total_tokens, H]        write strength
 *   gate        bf16  [total_tokens, H, d_v]   output-gate logits, or NULL for no gate
 *   A_log       fp32  [H]                      per-head log-scale A_h of the decay mapping
 *   cu_seqlens  int32 [num_seqs + 1]           device; 0 = cu[0] <= ... <= cu[num_seqs] = total_tokens
 *   initial_state fp32 [num_seqs, H, d_k, d_v] or NULL (zeros)
 *   final_state   fp32 [num_seqs, H, d_k, d_v] or NULL (not written); may alias initial_state
 *   out         [total_tokens, H, d_v] of out_dtype (bf16 or fp32)
 * max_seqlen: an upper bound on every sequence length, or 0 for none.  A sequence longer than a
 *   non-zero bound is reported through the error word (the result is still computed in full).
 * scale multiplies q.  workspace: device scratch of at least kda_chunk_fwd_workspace_min(...)
 *   bytes (equal to kda_chunk_fwd_workspace_size(...)), 256-byte aligned, or NULL when that size is
 *   0; its contents need no initialisation and it may be reused across calls on one stream.
 * Two kernels compute the same chunkwise form (kda_set_prefill_path below):
 *   - with d_k = d_v = 128 and at least a third as many (sequence, head) units as the GPU has SMs,
 *     one CTA per unit keeps every chunk intermediate on chip and needs no workspace (size 0);
 *   - otherwise a unit's chunks are spread over d_v / 32 CTAs of a cluster, handing chunk records
 *     to each other through per-unit rings in the workspace (about 0.63 MiB per unit at d = 128).
 * Numerics: the decay arithmetic, the accumulation and the carried state are fp32; the tensor-core
 *   operands are tf32 (the 16-token diagonal Gram blocks) and fp16 (everything else).  Values,
 *   states and the chunk pseudo-values must therefore stay within +-65504 (unit-norm q and k and
 *   O(1) values are far inside); a call that leaves that range ends with a non-finite state, which
 *   kda_sync_check reports as KDA_ERR_RANGE.
 * A zero-length sequence copies its initial state (or zeros) to final_state.
 * total_tokens == 0 or num_seqs == 0 is valid and only writes final_state.
 */
KDA_API kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const void *a,
                         const float *beta, const void *gate, const float *A_log,
                         const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                         int32_t max_seqlen, int32_t H, int32_t d_k, int32_t d_v, float scale,
                         const float *initial_state, float *final_state, void *out,
                         kda_dtype out_dtype, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * kda_chunk_fwd_noalloc — kda_chunk_fwd for callers that cannot allocate device memory.
 * (No counterpart in the pages: this is a deployment convenience, not part of the method.)
 *
 * Some callers cannot hand the library a workspace: their device memory belongs to someone else
 * (a serving engine's pre-reserved pool, a runtime plugin whose enqueue path must not allocate),
 * or they cannot afford the implicit synchronisation of cudaMalloc on a latency-critical path.
 * This entry point takes the same arguments as kda_chunk_fwd minus the workspace and instead uses
 * scratch memory built into the library: a 32 MiB device array that every GPU which loads
 * libkda holds until the process exits.  It calls no cudaMalloc or cudaFree.
 *   - Every call looks up that array's device address (with the calling thread's current device);
 *     the first call on a device loads the library's device code there, so make it before any
 *     stream capture.
 *   - With d_k = d_v = 128 and the kernel left to the shapes (kda_set_prefill_path(0)), a call
 *     whose cluster-kernel records would exceed 32 MiB (more than 50 units) runs the per-unit
 *     kernel, which needs no scratch, so no such call is rejected.  Otherwise sizes whose scratch
 *     need (kda_chunk_fwd_workspace_min) exceeds 32 MiB are rejected with KDA_ERR_INVALID_ARG and a
 *     message in kda_last_error (forcing the cluster kernel, kda_set_prefill_path(1), allows 50
 *     units of d = 128).
 *   - Every call on a device shares the one array and nothing in it needs to start at zero, but
 *     calls that overlap on the GPU (different streams, or other threads) race on it: serialise
 *     them, for example by issuing them all on one stream.
 */
KDA_API kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const void *a,
                                         const float *beta, const void *gate, const float *A_log,
                                         const int32_t *cu_seqlens, int32_t num_seqs,
                                         int64_t total_tokens, int32_t max_seqlen, int32_t H,
                                         int32_t d_k, int32_t d_v, float scale,
                                         const float *initial_state, float *final_state, void *out,
                                         kda_dtype out_dtype, void *stream);

/*
 * kda_chunk_fwd_host — kda_chunk_fwd with every input and output in HOST memory (page-locked for
 * the copies to overlap): the end-to-end prefill of a batch that lives on the host.
 * (No counterpart in the pages: this is the runtime around the method.)
 *   q, k, v, a, beta, gate, out, initial_state, final_state: host pointers, layouts and types as
 *     kda_chunk_fwd; A_log fp32 [H] and cu_seqlens int32 [num_seqs + 1] are HOST arrays here (read
 *     by this call; cu_seqlens must run monotonically from 0 to total_tokens).
 *   piece_tokens: tokens per piece (0 = 2048; at least 64).
 *   device_buffer: caller-owned device memory, 256-byte aligned, of
 *     kda_chunk_fwd_host_buffer_size(...) bytes: two staging slots, the prefill workspace and the
 *     states.
 * The batch is cut into pieces along the packed token axis (the last piece cut again 3 : 1 so that
 * little is left to copy out at the end); a cut inside a sequence falls on a 64-token chunk
 * boundary of that sequence, so every piece runs the chunks the whole call would,
 * and a sequence that continues into the next piece hands its state over on the device.  The
 * host-to-device copy of piece i+1, the prefill of piece i (on `stream`) and the device-to-host
 * copy of piece i-1 run on three streams at once.  Asynchronous with respect to the host: the
 * host buffers must stay valid, and `out` / `final_state` hold the results, once `stream` has
 * reached the end of the call.
 */
KDA_API kda_status kda_chunk_fwd_host(const void *q, const void *k, const void *v, const void *a,
                                      const float *beta, const void *gate, const float *A_log,
                                      const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                      int32_t H, int32_t d_k, int32_t d_v, float scale,
                                      const float *initial_state, float *final_state, void *out,
                                      kda_dtype out_dtype, int64_t piece_tokens, void *device_buffer,
                                      size_t device_buffer_bytes, void *stream);

/* Device buffer kda_chunk_fwd_host needs (host-only; reads the host cu_seqlens; 0 on invalid
 * arguments). */
KDA_API size_t kda_chunk_fwd_host_buffer_size(const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                              int32_t H, int32_t d_k, int32_t d_v, kda_dtype out_dtype,
                                              int64_t piece_tokens);

/* Workspace kda_chunk_fwd needs for these sizes (host-only; 0 on invalid sizes). */
KDA_API size_t kda_chunk_fwd_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen,
                                    int32_t H, int32_t d_k, int32_t d_v);

/* Same value as kda_chunk_fwd_workspace_size (kept so callers can ask for the minimum by name). */
KDA_API size_t kda_chunk_fwd_workspace_min(int64_t total_tokens, int32_t num_seqs, int32_t max_seqlen,
                                   int32_t H, int32_t d_k, int32_t d_v);

/*
 * kda_decode_step — one recurrent step for N independent sequences, state updated in place
 * (the fixed-size decode state of "K3 Architecture Illustrated", FIG 22: the state's shape does
 * not grow with the context).
 *   q, k, a     bf16 [N, H, d_k]      v, gate bf16 [N, H, d_v] (gate may be NULL)
 *   beta        fp32 [N, H]           A_log fp32 [H]
 *   state       fp32 [N, H, d_k, d_v] read and overwritten with the new state
 *   out         [N, H, d_v] of out_dtype (bf16 or fp32)
 */
KDA_API kda_status kda_decode_step(const void *q, const void *k, const void *v, const void *a,
                           const float *beta, const void *gate, const float *A_log, float *state,
                           void *out, kda_dtype out_dtype, int32_t N, int32_t H, int32_t d_k,
                           int32_t d_v, float scale, void *stream);

/*
 * Multi-token decode with rollback (speculative decoding).  The pages state only that KDA's
 * recurrent state needs rollback handling after rejected proposals ("K3 Architecture
 * Illustrated", "Speculative decoding changes the value of extra computation"); these two calls
 * are the plainest reading: verify K proposed tokens, then keep the state of the accepted prefix.
 *
 * kda_decode_verify — runs tokens 1..K of each of N sequences from its current state, exactly as K
 * calls of kda_decode_step would, but does not write the state.  For every token it writes the
 * output and the write vector u_t = beta_t (v_t - (Diag(alpha_t) S_{t-1})^T k_t).
 *   q, k, a     bf16 [N, K, H, d_k]      v, gate bf16 [N, K, H, d_v] (gate may be NULL)
 *   beta        fp32 [N, K, H]           A_log fp32 [H]
 *   state       fp32 [N, H, d_k, d_v]    read only
 *   u           fp32 [N, H, K, d_v]      written (consumed by kda_decode_commit)
 *   out         [N, K, H, d_v] of out_dtype
 * 1 <= K <= 16.  The caller owns every buffer.
 */
KDA_API kda_status kda_decode_verify(const void *q, const void *k, const void *v, const void *a,
                                     const float *beta, const void *gate, const float *A_log,
                                     const float *state, float *u, void *out, kda_dtype out_dtype,
                                     int32_t N, int32_t K, int32_t H, int32_t d_k, int32_t d_v,
                                     float scale, void *stream);

/*
 * kda_decode_commit — advances state n by its first accepted[n] verified tokens:
 *   S <- Diag(alpha_t) S + k_t u_t^T  for t = 1 .. accepted[n]
 * with the same k, a, A_log and K as the verify call and its u.  accepted (int32 [N], device)
 * must lie in [0, K]; 0 leaves a state untouched.  A count outside [0, K] is clamped and reported
 * through the error word (kda_sync_check returns KDA_ERR_INVALID_ARG).
 */
KDA_API kda_status kda_decode_commit(const void *k, const void *a, const float *A_log,
                                     const int32_t *accepted, const float *u, float *state,
                                     int32_t N, int32_t K, int32_t H, int32_t d_k, int32_t d_v,
                                     void *stream);

/*
 * The module pieces around the recurrence.  The pages say only that the actual KDA module also has
 * short convolution, normalisation and output gating ("K3 Architecture Illustrated", FIG 21) and
 * that short convolution depends on input order (§"Why can K3's MLA use NoPE?"); the forms below
 * are the plainest readings.
 *
 * kda_short_conv — causal depthwise convolution over time, per sequence of the packed batch:
 *   y_t[h][c] = sum_{j < width} w[h][c][j] * x_{t-(width-1)+j}[h][c]     (x before a sequence = 0)
 * optionally followed (l2norm != 0) by y_t[h] <- y_t[h] / sqrt(|y_t[h]|^2 + 1e-12).
 *   x, y  bf16 [total_tokens, H, d] (d = 64 or 128; y may not alias x)
 *   w     fp32 [H, d, width], 1 <= width <= 4
 *   cu_seqlens int32 [num_seqs + 1] (device), as for kda_chunk_fwd.
 * Malformed cu_seqlens are reported through the error word.
 */
KDA_API kda_status kda_short_conv(const void *x, const float *w, const int32_t *cu_seqlens, int32_t num_seqs,
                                  int64_t total_tokens, int32_t H, int32_t d, int32_t width, int32_t l2norm,
                                  void *y, void *stream);

/*
 * kda_output_norm_gate — pre-gate RMS normalisation of every (token, head) output row, then the
 * sigmoid output gate:  out = sigmoid(gate) * o / sqrt(mean_c(o^2) + eps) * w.
 *   o     fp32 [total_tokens, H, d_v] (e.g. kda_chunk_fwd with gate = NULL and fp32 output)
 *   gate  bf16 [total_tokens, H, d_v] or NULL (no gate)
 *   w     fp32 [d_v] per-channel gain, shared by the heads
 *   out   [total_tokens, H, d_v] of out_dtype
 */
KDA_API kda_status kda_output_norm_gate(const float *o, const void *gate, const float *w, int64_t total_tokens,
                                        int32_t H, int32_t d_v, float eps, void *out, kda_dtype out_dtype,
                                        void *stream);

/*
 * kda_state_combine — one affine state map per (sequence, head) unit, for context-parallel prefill
 * (a sequence split into segments held by different GPUs):
 *   S_out[u] = M[u] S_in[u] + B[u]
 *   M fp32 [units, d_k, d_k]; S_in, B, S_out fp32 [units, d_k, d_v]; S_out may alias B, not S_in.
 * Over a segment, the recurrence maps its incoming state S to M S + B, where B is the state it
 * reaches from S = 0 and M the state the homogeneous recurrence (v = 0) reaches from S = I; both
 * come from kda_chunk_fwd (the pages carry the state sequentially from chunk to chunk: "Kimi K3 ·
 * Lesson 3 of 14", CHUNKWISE diagram).  At most 65535 units per call.
 */
KDA_API kda_status kda_state_combine(const float *M, const float *S_in, const float *B, float *S_out,
                                     int32_t units, int32_t d_k, int32_t d_v, void *stream);

/*
 * kda_segment_maps — the affine map S -> M S + B of every (sequence, head) unit over the tokens
 * given (the maps kda_state_combine folds), in one pass: the recurrence is linear in (v, S) column
 * by column, so [M | B] is the final state of one run over the value columns [0 | v] from the
 * initial state [I | 0], and the chunk-local work (decays, Gram blocks, triangular solve, W) is
 * shared by both maps.  (Context-parallel prefill; "Kimi K3 · Lesson 3 of 14", CHUNKWISE diagram:
 * the state passes from chunk to chunk, here from segment to segment.)
 *   q, k, a, v bf16 [total_tokens, H, d] (d_k = d_v = d, 64 or 128); beta fp32 [total_tokens, H];
 *   A_log fp32 [H]; cu_seqlens int32 [num_seqs + 1] on the device, as kda_chunk_fwd;
 *   M, B fp32 [num_seqs, H, d, d] (written; caller-owned).
 *   workspace: kda_segment_maps_workspace_size(...) bytes, 256-byte aligned, caller-owned.
 * Runs the cluster prefill kernel with 2d value columns (no outputs, no gate), then two strided
 * device copies.  Errors as kda_chunk_fwd; KDA_ERR_UNSUPPORTED for other d.
 */
KDA_API kda_status kda_segment_maps(const void *q, const void *k, const void *v, const void *a, const float *beta,
                                    const float *A_log, const int32_t *cu_seqlens, int32_t num_seqs,
                                    int64_t total_tokens, int32_t max_seqlen, int32_t H, int32_t d, float scale,
                                    float *M, float *B, void *workspace, size_t workspace_bytes, void *stream);

/* Workspace of kda_segment_maps (host-only; 0 on invalid sizes or unsupported d). */
KDA_API size_t kda_segment_maps_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d);

/*
 * kda_chunk_bwd — gradients of the prefill (kda_chunk_fwd with the same inputs) with respect to
 * q, k, v, the decay logits a, beta, the gate logits, A_log and the initial state, given dout (the
 * gradient of the outputs) and optionally dfinal_state (the gradient of the final states).  The
 * pages describe only the forward recurrence; this is its reverse-mode derivative, token by token
 * ("Review A · Sequence and depth", Free recall; "Kimi K3 · Lesson 3 of 14", eq. 5 passage).
 *   inputs      as kda_chunk_fwd (bf16 q, k, a, v, gate; fp32 beta, A_log; cu_seqlens on the device)
 *   dout        fp32 [total_tokens, H, d_v]        dfinal_state fp32 [num_seqs, H, d_k, d_v] or NULL
 *   dq, dk, da  fp32 [total_tokens, H, d_k]        dv, dgate fp32 [total_tokens, H, d_v]
 *   dbeta       fp32 [total_tokens, H]             dA_log fp32 [H] (overwritten: summed over sequences)
 *   dinitial_state fp32 [num_seqs, H, d_k, d_v] or NULL
 *   dgate must be given when gate is; workspace of kda_chunk_bwd_workspace_size(...) bytes, 16-byte
 *   aligned: the state at the start of every 32-token chunk plus a 32-state scratch per unit.
 * Runs a cluster of d_v / 32 CTAs per (sequence, head) (one per 32 value columns) over the tokens
 * in order, then in reverse: its time is the latency of the sequence's token steps.  Deterministic
 * except dA_log, which is summed with atomics over sequences and column slices.
 */
KDA_API kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const void *a, const float *beta,
                                 const void *gate, const float *A_log, const int32_t *cu_seqlens,
                                 int32_t num_seqs, int64_t total_tokens, int32_t H, int32_t d_k, int32_t d_v,
                                 float scale, const float *initial_state, const float *dout,
                                 const float *dfinal_state, float *dq, float *dk, float *dv, float *da,
                                 float *dbeta, float *dgate, float *dA_log, float *dinitial_state,
                                 void *workspace, size_t workspace_bytes, void *stream);

/*
 * kda_chunk_bwd_chunkwise — the same gradients as kda_chunk_bwd (same arguments and layouts), in
 * chunkwise form: per 64-token chunk the forward operands, the states at the chunk starts (a pass
 * over chunks), the state gradients at the chunk ends (a reverse pass over chunks) and the rest of
 * the gradients chunk by chunk, all in fp32; T / 64 sequential steps per unit instead of 3 T.
 * Workspace: kda_chunk_bwd_chunkwise_workspace_size(...) bytes, 16-byte aligned.
 */
KDA_API kda_status kda_chunk_bwd_chunkwise(const void *q, const void *k, const void *v, const void *a,
                                           const float *beta, const void *gate, const float *A_log,
                                           const int32_t *cu_seqlens, int32_t num_seqs, int64_t total_tokens,
                                           int32_t H, int32_t d_k, int32_t d_v, float scale,
                                           const float *initial_state, const float *dout,
                                           const float *dfinal_state, float *dq, float *dk, float *dv,
                                           float *da, float *dbeta, float *dgate, float *dA_log,
                                           float *dinitial_state, void *workspace, size_t workspace_bytes,
                                           void *stream);

/* Workspace of kda_chunk_bwd_chunkwise (host-only; 0 on invalid sizes): one record of the chunk's
 * operands, states and state gradients per (64-token chunk, head), (total_tokens / 64 + num_seqs)
 * x H records of 410,112 bytes at d_k = d_v = 128 (196,864 at 64): 1.69 GB for 8192 tokens x 32
 * heads, 215 GB for one 1 M-token sequence x 32 heads, more than one B200 holds -- use kda_chunk_bwd
 * (66 KiB per 32 tokens and head) for long sequences.  Deterministic except dA_log, which is summed
 * with float atomics over chunks, so its last bits can vary between runs. */
KDA_API size_t kda_chunk_bwd_chunkwise_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H,
                                                      int32_t d_k, int32_t d_v);

/* Workspace kda_chunk_bwd needs (host-only; 0 on invalid sizes):
 * ((total_tokens / 32 + num_seqs) * H + num_seqs * H * 32) * d_k * d_v * 4 bytes. */
KDA_API size_t kda_chunk_bwd_workspace_size(int64_t total_tokens, int32_t num_seqs, int32_t H, int32_t d_k,
                                            int32_t d_v);

/* Static description of a status code. */
KDA_API const char *kda_status_string(kda_status status);

/*
 * Synchronises `stream`, then reads and clears the current device's error word.  Returns
 * KDA_ERR_CUDA if the stream reported a CUDA error, KDA_ERR_INVALID_ARG if a kernel found
 * malformed cu_seqlens, a sequence longer than max_seqlen or an accepted count outside [0, K],
 * KDA_ERR_TIMEOUT if a bounded wait gave up, else KDA_OK.
 */
KDA_API kda_status kda_sync_check(void *stream);

/* Text of the most recent error seen by this thread's calls (never NULL; "" when none). */
KDA_API const char *kda_last_error(void);

/* Number of CUDA kernels this process has launched through libkda so far (all devices). */
KDA_API uint64_t kda_launch_count(void);

/*
 * kda_set_prefill_path — choose which of the two prefill kernels kda_chunk_fwd (and
 * kda_chunk_fwd_noalloc, kda_chunk_fwd_host) run for d_k = d_v = 128.  (No counterpart in the pages:
 * both kernels compute the same chunkwise form of "Kimi K3 · Lesson 3 of 14"; they differ only in how
 * the work is spread over the GPU.)
 *   path 0: chosen from the shapes (the default): one CTA per (sequence, head) unit when the units
 *           are more than twice the clusters of the cluster kernel that fit on the device at once
 *           (queried once with cudaOccupancyMaxActiveClusters: 33 on a 148-SM B200, so more than
 *           66 units), else the cluster kernel;
 *   path 1: the cluster kernel (a unit's chunks spread over d_v/32 CTAs, chunk records in the
 *           caller's workspace);
 *   path 2: one CTA per unit, every intermediate on chip (no workspace).
 * Other d_k, d_v always use the cluster kernel.  Process-wide; not synchronised with launches in
 * flight on other threads.  Returns KDA_ERR_INVALID_ARG for any other value.  The workspace size
 * (kda_chunk_fwd_workspace_size) follows the path in force when it is queried: 0 for path 2.
 */
KDA_API kda_status kda_set_prefill_path(int32_t path);

/* kda_prefill_path — the kernel kda_chunk_fwd would run for num_units (sequence, head) units of
 * this shape under the current setting: 1 (cluster kernel) or 2 (one CTA per unit). */
KDA_API int32_t kda_prefill_path(int64_t num_units, int32_t d_k, int32_t d_v);

/*
 * kda_inject_stall — failure injection for tests of the bounded waits.  (No counterpart in the
 * pages: the method has no inter-CTA waits; this exercises the library's own failure handling.)
 *
 * enable != 0: every later prefill launch in this process (kda_chunk_fwd, kda_chunk_fwd_noalloc)
 *   withholds the publication of chunk 0 of every (sequence, head) unit, so the waits on it can
 *   never be satisfied, and every device-side wait gives up after wait_limit_ns nanoseconds
 *   (1e6 <= wait_limit_ns <= 4e9, else KDA_ERR_INVALID_ARG).  Such a call still returns KDA_OK;
 *   its outputs are undefined, and the following kda_sync_check returns KDA_ERR_TIMEOUT.  The
 *   CUDA context stays usable.
 * enable == 0: back to normal operation (wait_limit_ns is ignored; the bound returns to 4 s).
 * Process-wide; not synchronised with launches in flight on other threads.
 */
KDA_API kda_status kda_inject_stall(int32_t enable, uint64_t wait_limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* KDA_H_ */
