/*
 * kda.h -- C ABI of the B200 (sm_100a) Kimi Delta Attention (KDA) library.
 *
 * The token mixer (Kimi Linear paper notes, paper-notes-site, section 2,
 * KDA recurrence equation; the bullet between the terms read as "+"):
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * per (sequence, head), with an fp32 state S of shape dk x dv (row c = key
 * channel c) and a per-channel decay alpha_t = exp(g_t).  Two entry points:
 *
 *   kda_chunk_fwd       prefill: the chunkwise-parallel form (chunk C = 64)
 *                       of the paper notes, section 3 (old-state contribution
 *                       through the chunk's transitions plus the intra-chunk
 *                       writes, via a WY-like W,U representation);
 *   kda_recurrent_step  decode: one token per sequence, the fused recurrent
 *                       form the same section names for short queries;
 *   kda_recurrent_steps decode for serving: up to L tokens per sequence
 *                       (short queries) on a slot-indexed state pool;
 *   kda_chunk_fwd_host  kda_chunk_fwd on host buffers, copies pipelined
 *                       against the computation;
 *   kda_gated_rmsnorm   the output epilogue (RMSNorm with a sigmoid gate).
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers (cudaMalloc'd or any memory the
 *     device can address), contiguous, row-major, 16-byte aligned (beta,
 *     cu_seqlens and slots: 4-byte aligned).  The
 *     caller allocates and owns every buffer; the library keeps no pointer
 *     after a call returns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued on it and the call returns without synchronising.
 *   - g is log(alpha) (fp32, any finite value <= 0 is a decay; see the
 *     per-function numerical range), beta is fp32.  q is used as given: no
 *     scale, L2 norm, gate or sigmoid is applied inside.
 *   - Argument errors return synchronously and enqueue nothing.  A failed
 *     launch returns KDA_ERR_CUDA.  Conditions detected on the device (a
 *     bounded wait that ran out) set a per-device error word that
 *     kda_get_device_error() reports; no kernel traps.
 *   - kda_last_error_message() gives a human-readable detail of the calling
 *     thread's last failing call.
 */
#ifndef KDA_B200_H
#define KDA_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    KDA_OK = 0,
    KDA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, bad offsets */
    KDA_ERR_UNSUPPORTED = 2,  /* valid but not implemented (dk, dv, dtype) */
    KDA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    KDA_ERR_DEVICE = 4        /* the device error word was set */
} kda_status;

typedef enum {
    KDA_F32 = 0,   /* q, k, v, out are float32 */
    KDA_BF16 = 1   /* q, k, v, out are bfloat16 */
} kda_dtype;

/*
 * Input prologue flags of the *_ex calls (and kda_recurrent_steps), applied
 * inside the kernels before the method runs, per (token, head):
 *   KDA_QK_L2NORM     q <- q / |q|_2 and k <- k / |k|_2 (fp32; a zero vector
 *                     stays zero)
 *   KDA_BETA_SIGMOID  beta <- 1 / (1 + exp(-beta))  (beta given as a logit)
 * and then q <- q_scale * q.  flags = 0 with q_scale = 1 is the identity.
 * Source: Kimi Linear paper notes (paper-notes-site), section 7: the open
 * layer hands raw projections to the KDA kernels with the q/k L2 norm done
 * inside the kernel (use_qk_l2norm_in_kernel) and takes beta as the sigmoid
 * of a projection; the gate activation (A_log, dt_bias) is not on the pages
 * and is not offered.
 */
enum { KDA_QK_L2NORM = 1, KDA_BETA_SIGMOID = 2 };
/* kda_recurrent_steps only: compute the L tokens in the chunk form on tensor
 * cores (see kda_recurrent_steps). */
enum { KDA_STEPS_CHUNK = 4 };

/*
 * kda_chunk_fwd -- prefill forward over whole sequences.
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 2 (recurrence)
 * and section 3 (chunkwise parallel form; the layer passes initial_state and
 * receives the final recurrent state); the whoami-wesleyyou blog, "context
 * modification and checkpoint" section (a state is the checkpoint of its
 * prefix: resuming from it continues the recurrence exactly).
 *
 * Layout (dense mode, cu_seqlens == NULL; N = B sequences of length T):
 *   q, k   [B, T, H, dk]  dtype        v    [B, T, H, dv]  dtype
 *   g      [B, T, H, dk]  float32      beta [B, T, H]      float32
 *   out    [B, T, H, dv]  dtype (written, rounded to nearest even for bf16)
 *   initial_state [N, H, dk, dv] float32, or NULL for zeros
 *   final_state   [N, H, dk, dv] float32, or NULL to skip; it may equal
 *                 initial_state (in-place resume)
 * Varlen mode (cu_seqlens != NULL): B must be 1; cu_seqlens is a device
 *   int32 array [num_seqs + 1] with cu[0] = 0, non-decreasing, cu[num_seqs] =
 *   T; sequence n is tokens [cu[n], cu[n+1]).  Zero-length sequences are
 *   allowed (final = initial).  The offsets are read on the device; they are
 *   not validated there beyond clamping to [0, T].
 *   In dense mode num_seqs is ignored (N = B).
 *
 * Supported: dtype KDA_BF16 with dk = dv = 128 (tensor-core path), and
 *   KDA_F32 with dk, dv in {64, 128} (exact fp32 path).  Others return
 *   KDA_ERR_UNSUPPORTED.
 * Numerical range (bf16 path): any finite per-token g <= 0, and g <= 5 for
 *   positive gates.  A chunk whose decay over its 64 tokens stays within
 *   e^{+-80} references its exponents at the chunk start (the fast path);
 *   any other chunk references them per 16-token sub-chunk, inside the same
 *   call, and a sub-chunk whose own decay falls below 2^-60 has its diagonal
 *   blocks formed from e^{G_i - G_j} directly; the result is the same up to
 *   rounding.
 * Aliasing: out must not overlap any input.
 * Memory: the bf16 path takes a stream-ordered scratch buffer from a
 *   library-private pool on the current device (cudaMallocFromPoolAsync on
 *   `stream`), freed stream-ordered before the call returns; the pool keeps
 *   the memory for reuse by later calls.
 */
kda_status kda_chunk_fwd(const void *q, const void *k, const void *v,
                         const float *g, const float *beta,
                         const float *initial_state, const int32_t *cu_seqlens,
                         void *out, float *final_state,
                         int B, int T, int H, int dk, int dv, int num_seqs,
                         kda_dtype dtype, void *stream);

/*
 * kda_chunk_fwd_ex -- kda_chunk_fwd with the input prologue (flags, q_scale;
 * see KDA_QK_L2NORM).  Same arguments, layouts and support otherwise;
 * unknown flag bits or a non-finite q_scale return KDA_ERR_INVALID_ARG.
 */
kda_status kda_chunk_fwd_ex(const void *q, const void *k, const void *v,
                            const float *g, const float *beta,
                            const float *initial_state, const int32_t *cu_seqlens,
                            void *out, float *final_state,
                            int B, int T, int H, int dk, int dv, int num_seqs,
                            kda_dtype dtype, unsigned flags, float q_scale, void *stream);

/*
 * kda_chunk_fwd_host -- kda_chunk_fwd on HOST buffers, with the host<->device
 * copies pipelined against the computation.
 *
 * Source: as kda_chunk_fwd; the pipelining rests on the checkpoint semantics
 * (whoami-wesleyyou blog, "context modification and checkpoint": a state
 * summarises its prefix exactly) -- the packed token axis is processed in
 * ranges, each range resuming its sequences from the fp32 states the
 * previous range left on the device.  A range ends at a sequence end or a
 * whole number of chunks into a sequence, so every sequence keeps the chunk
 * grid, and the result, of one kda_chunk_fwd call.  The pages have no
 * host-buffer entry point; this is a deployment variant.
 *
 * Pointers: q, k, v, g, beta, initial_state (nullable), out, final_state
 *   (nullable) are HOST pointers with kda_chunk_fwd's layouts (dense [B, T,
 *   H, *], or varlen [1, T, H, *] with states [num_seqs, H, dk, dv]).
 *   cu_seqlens (nullable = dense mode) is a HOST int32 array [num_seqs + 1],
 *   checked in full (cu[0] = 0, non-decreasing, cu[num_seqs] = T; else
 *   KDA_ERR_INVALID_ARG).  Page-locked (pinned) memory lets the copies
 *   overlap the computation; pageable memory works, with copies that do not
 *   overlap.
 * range_tokens: tokens per pipeline stage, rounded up to a multiple of 64;
 *   0 selects 2048 (measured best for 32 heads x d = 128 over PCIe).
 * Streams: the computation runs on `stream`; the copies run on two streams
 *   the library keeps per device, ordered after the work already queued on
 *   `stream`, and `stream` is ordered after them, so the outputs are in host
 *   memory once `stream` has completed (e.g. cudaStreamSynchronize).
 * Memory: device buffers for two input stages, two output stages, every
 *   sequence's state and the ranges' offsets come from the library-private
 *   pool (stream-ordered, as in kda_chunk_fwd) and are released on `stream`.
 * Supported: as kda_chunk_fwd.
 * Aliasing: out and final_state must not overlap any input.
 */
kda_status kda_chunk_fwd_host(const void *q, const void *k, const void *v,
                              const float *g, const float *beta,
                              const float *initial_state, const int32_t *cu_seqlens,
                              void *out, float *final_state,
                              int B, int T, int H, int dk, int dv, int num_seqs,
                              kda_dtype dtype, int range_tokens, void *stream);

/*
 * kda_recurrent_step -- one decode token for each of N sequences.
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 2 (recurrence)
 * and section 3 (the fused recurrent mode used for short queries outside
 * training: only the recurrent state is kept).
 *
 * Layout: q, k [N, H, dk] dtype; v [N, H, dv] dtype; g [N, H, dk] float32;
 *   beta [N, H] float32; state_inout [N, H, dk, dv] float32, read and
 *   overwritten in place with S_t; out [N, H, dv] dtype.
 * Computes a = exp(g); S' = Diag(a) S; u = beta (v - S'^T k);
 *   S = S' + k u^T; o = S^T q, reading and writing each state once.
 * Supported: dk, dv in {64, 128}, dtype KDA_BF16 or KDA_F32.  Any finite g.
 * Aliasing: out must not overlap any input; state_inout must not overlap
 *   the token inputs.
 */
kda_status kda_recurrent_step(const void *q, const void *k, const void *v,
                              const float *g, const float *beta,
                              float *state_inout, void *out,
                              int N, int H, int dk, int dv,
                              kda_dtype dtype, void *stream);

/*
 * kda_recurrent_step_ex -- kda_recurrent_step with the input prologue
 * (flags, q_scale; see KDA_QK_L2NORM).  Unknown flag bits or a non-finite
 * q_scale return KDA_ERR_INVALID_ARG.
 */
kda_status kda_recurrent_step_ex(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 float *state_inout, void *out,
                                 int N, int H, int dk, int dv,
                                 kda_dtype dtype, unsigned flags, float q_scale,
                                 void *stream);

/*
 * kda_recurrent_steps -- L decode tokens for each of N sequences whose states
 * live in a slot-indexed pool (continuous batching).
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 2 (recurrence)
 * and section 3 (queries of at most 64 tokens outside training take the
 * fused recurrent mode, which keeps only the recurrent state); section 7
 * (the serving-side wrapper owns the state's dtype and shape).  The slot
 * array itself is a serving layout with no counterpart in the pages.
 *
 * Layout: q, k [N, L, H, dk] dtype; v [N, L, H, dv] dtype; g [N, L, H, dk]
 *   float32; beta [N, L, H] float32; out [N, L, H, dv] dtype;
 *   state_pool [num_slots, H, dk, dv] float32; slots: device int32 [N] or
 *   NULL (sequence n uses pool entry n, which needs num_slots >= N).
 * Computes, for each sequence n and head, the L steps of kda_recurrent_step
 *   in order on pool entry slots[n], reading the state once and writing it
 *   once (L tokens cost one state read and one write, not L of each).
 * Errors: a slot outside [0, num_slots) skips that sequence (its pool entry
 *   and outputs are not written) and sets the device error word, reported by
 *   kda_get_device_error with code 3.  Slots must be distinct: two sequences
 *   naming one entry race.  L >= 1 (the paper's mode switch is at 64 tokens;
 *   longer inputs belong to kda_chunk_fwd, but any L is computed correctly).
 * Prologue: flags and q_scale as in the *_ex calls (KDA_QK_L2NORM); pass
 *   0 and 1.0f for inputs that are already normalised.
 * Supported: dk, dv in {64, 128}, dtype KDA_BF16 or KDA_F32.  Any finite g.
 * Aliasing: out must not overlap any input; the pool must not overlap the
 *   token inputs.
 */
/*
 * KDA_STEPS_CHUNK in flags selects, for dtype KDA_BF16 with dk = dv = 128,
 * L >= 2 and no prologue flags (q_scale = 1), the chunk form of the same L
 * steps (section 3 of the notes: a WY-like representation of the block's
 * writes, then one product with the state) on tensor cores: blocks of 16
 * tokens up to L = 32; from L = 33 on, 64-token chunks on tcgen05 with the
 * intra-chunk work and the state product fused per (sequence, head) (when
 * state_pool and out are 32-byte aligned; else the 16-token blocks).  The
 * operands of the state products (state, V_new, T, P and the decayed k, q)
 * are rounded to bf16 as in kda_chunk_fwd, the state stays fp32.  Any
 * finite g <= 0, and g <= 5 for positive gates (a 64-token chunk whose decay
 * leaves e^{+-80} is finished in 16-token blocks).  The 64-token path takes
 * a scratch of 32 KB per SM plus 8 bytes per (sequence, head) from the
 * library's stream-ordered memory pool, released on the stream before the
 * call returns.  Other combinations run the recurrent kernel, which is
 * bitwise equal to L calls of kda_recurrent_step.
 */
kda_status kda_recurrent_steps(const void *q, const void *k, const void *v,
                               const float *g, const float *beta,
                               float *state_pool, const int32_t *slots, int num_slots,
                               void *out, int N, int L, int H, int dk, int dv,
                               kda_dtype dtype, unsigned flags, float q_scale,
                               void *stream);

/*
 * kda_gated_rmsnorm -- the layer's output epilogue: an RMSNorm with a
 * sigmoid output gate, per row of dv values.
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 7: the layer
 * passes the KDA readout through FusedRMSNormGated (sigmoid output gate)
 * before the output projection.
 *
 * Computes, for each of `rows` rows (e.g. rows = B * T * H of the prefill
 * output [B, T, H, dv], or N * H of a decode output):
 *     out = x / sqrt(mean(x^2) + eps) * weight * 1 / (1 + exp(-gate))
 * in fp32, rounded to nearest even for bf16.
 * Layout: x, gate, out [rows, dv] dtype (device, 16-byte aligned); weight
 *   [dv] float32 (device).  out may equal x (in place); it must not overlap
 *   gate or weight otherwise.
 * Supported: dv in {64, 128}, dtype KDA_BF16 or KDA_F32; eps finite >= 0.
 */
kda_status kda_gated_rmsnorm(const void *x, const void *gate, const float *weight,
                             float eps, void *out, long long rows, int dv,
                             kda_dtype dtype, void *stream);

/*
 * kda_recurrent_bwd -- gradients of kda_chunk_fwd's result (dense layout),
 * for training.
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 2 (the
 * recurrence) and section 3 (training takes the chunked kernels and their
 * backward); the backward is the chain rule through the recurrence:
 *   dS += q do^T;  dq = S_t do;  du = dS^T k;  dk = dS u + S' dw (dw = -beta du);
 *   dbeta = du . (v - w);  dv = beta du;  dS' = dS + k dw^T;
 *   dg = rowsum(dS' o S');  dS_{t-1} = Diag(exp g) dS'
 *   with S' = Diag(exp g) S_{t-1}, w = S'^T k, u = beta (v - w), S_t = S' + k u^T,
 * starting from dS_T = dfinal_state (or 0) and ending at dinitial_state.
 *
 * Layout: q, k [B, T, H, dk] dtype; v, dout [B, T, H, dv] dtype; g
 *   [B, T, H, dk] float32; beta [B, T, H] float32; initial_state,
 *   dfinal_state [B, H, dk, dv] float32 or NULL (zeros).  Outputs, float32,
 *   written in full: dq, dk, dg [B, T, H, dk]; dv [B, T, H, dv]; dbeta
 *   [B, T, H]; dinitial_state [B, H, dk, dv] or NULL (not written).
 * Computation: one warp per (sequence, head, 16-column tile of the state) in
 *   fp32: a forward pass storing the state every 8 tokens, then blocks in
 *   reverse with the block's states recomputed; per-tile partial row sums
 *   reduced by a second kernel in a fixed order (deterministic).  Workspace
 *   from the device's stream-ordered pool on `stream`.
 * Supported: dk, dv in {64, 128}; dtype KDA_BF16 or KDA_F32; dense only (no
 *   cu_seqlens); no prologue flags.  Pointers 16-byte aligned (beta, dbeta 4).
 */
kda_status kda_recurrent_bwd(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *initial_state, const void *dout,
                             const float *dfinal_state, float *dq, float *dk, float *dv,
                             float *dg, float *dbeta, float *dinitial_state, int B, int T, int H,
                             int dk_, int dv_, kda_dtype dtype, void *stream);

/*
 * kda_chunk_bwd -- gradients of kda_chunk_fwd's result by the chunked form on
 * the tensor cores, for training (bf16, dk = dv = 128).
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 3 (training
 * takes the chunked kernels and their backward); the equations are reverse
 * mode through the chunk form of section 3 (derived from the section 2
 * recurrence).  Per chunk, S the state entering it and dS' the gradient of
 * the state leaving it (dS' = dfinal_state, or 0, for the last chunk):
 *   dV_new = P^T dO + Kt dS',  dS = Qg^T dO + Diag(e^{G_C}) dS' - W^T dV_new
 * (last chunk first), then per chunk dP = tril0(dO V_new^T), dKt = V_new dS'^T,
 *   dW = -dV_new S^T, dT = dV_new (beta V)^T + dW (beta K e^G)^T,
 *   dA = tril_-1(-T^T dT T^T), and the gradients of the decayed forms down to
 *   dq, dk, dv, dbeta and dg (the in-chunk reverse cumsum of dG).
 * Computation: the forward prep and chain recomputed (the chain also storing
 *   S and V_new per chunk as bf16), a reverse chain over chunks per (sequence,
 *   head, 32-column tile), and one CTA per (chunk, head) for the rest; bf16
 *   tensor-core operands, fp32 accumulation and state gradient.  Workspace
 *   from the device's stream-ordered pool on `stream`: 168.5 KiB per (chunk,
 *   head).
 * Layout: as kda_chunk_fwd for q, k, v, g, beta, initial_state, cu_seqlens
 *   (varlen: B == 1, num_seqs sequences); dout [B, T, H, dv] bf16;
 *   dfinal_state, dinitial_state [N, H, dk, dv] float32 or NULL (zeros / not
 *   written).  Outputs, float32, written for every token: dq, dk, dg
 *   [B, T, H, dk]; dv [B, T, H, dv]; dbeta [B, T, H].
 * Range: a chunk in which some |G| or G_C - G exceeds 80 (an average per-token
 *   log-decay below -1.25 on a channel over 64 tokens) sets the device error
 *   word (kda_get_device_error returns KDA_ERR_DEVICE) and its gradients are
 *   not written; kda_recurrent_bwd covers such inputs.
 * Supported: KDA_BF16 with dk = dv = 128 (else KDA_ERR_UNSUPPORTED).
 *   Pointers 16-byte aligned (beta, dbeta, cu_seqlens 4).
 */
kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *initial_state,
                         const int32_t *cu_seqlens, const void *dout, const float *dfinal_state,
                         float *dq, float *dk, float *dv, float *dg, float *dbeta,
                         float *dinitial_state, int B, int T, int H, int dk_, int dv_,
                         int num_seqs, kda_dtype dtype, void *stream);

/*
 * kda_chunk_fwd_save, kda_chunk_bwd_saved -- a training step that keeps the
 * forward's intermediates for the backward instead of recomputing them.
 *
 * Source: Kimi Linear paper notes (paper-notes-site), section 3: the chunked
 * forward used in training saves its intermediates (the decay cumsum, the
 * A/P blocks, w, u, the decayed q and k, v_new and the chunk states) so
 * that the backward can use them; the same role here is played by the
 * per-(chunk, head) records, the bf16 state entering each chunk and V_new.
 *
 * kda_chunk_saved_bytes: bytes of the intermediates for a call of these
 *   sizes (varlen = 0: dense [B, T]; varlen = 1: B == 1 and num_seqs
 *   sequences); -1 for bad sizes.  About 122 KB per (64-token chunk, head):
 *   500 MB for T = 8192, H = 32.
 * kda_chunk_fwd_save: kda_chunk_fwd (same arguments, layouts, results;
 *   KDA_BF16 with dk = dv = 128 only) that also writes the intermediates into
 *   `saved` (device memory, 256-byte aligned, at least saved_bytes >=
 *   kda_chunk_saved_bytes; the caller owns it).  It allocates nothing.
 * kda_chunk_bwd_saved: kda_chunk_bwd (same arguments and results) given the
 *   `saved` buffer of a kda_chunk_fwd_save call on the SAME inputs,
 *   initial_state and cu_seqlens (nothing checks this; other contents give
 *   wrong gradients); it skips recomputing the forward.  The gradients are
 *   bitwise equal to kda_chunk_bwd's.  Scratch for the reverse chain's
 *   images (48 KB per (chunk, head)) comes from the library pool.
 * Errors: as kda_chunk_fwd / kda_chunk_bwd, plus KDA_ERR_INVALID_ARG for a
 *   null, misaligned or too small `saved`.
 */
long long kda_chunk_saved_bytes(int B, int T, int H, int num_seqs, int varlen);
kda_status kda_chunk_fwd_save(const void *q, const void *k, const void *v,
                              const float *g, const float *beta,
                              const float *initial_state, const int32_t *cu_seqlens,
                              void *out, float *final_state,
                              int B, int T, int H, int dk, int dv, int num_seqs,
                              kda_dtype dtype, void *saved, long long saved_bytes, void *stream);
kda_status kda_chunk_bwd_saved(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, const float *initial_state,
                               const int32_t *cu_seqlens, const void *dout,
                               const float *dfinal_state, float *dq, float *dk, float *dv,
                               float *dg, float *dbeta, float *dinitial_state, int B, int T,
                               int H, int dk_, int dv_, int num_seqs, kda_dtype dtype,
                               const void *saved, long long saved_bytes, void *stream);

/*
 * kda_state_affine -- S_out = M S_in + B for `count` independent blocks.
 *
 * Source: the recurrence of the paper notes (section 2) is affine in the
 * state: a segment of tokens maps any start state S to M S + B, with B the
 * segment's final state from S = 0 and M its final state from S = I with
 * v = 0.  This call composes such maps, the exchange step of a sequence
 * split across devices (gated_delta_rule_88_b200.cp); the pages describe no
 * multi-device prefill.
 *
 * Layout: M [count, dk, dk]; B (nullable = 0), S_in, S_out [count, dk, dv];
 *   float32 device memory, 4-byte aligned.  S_out must not overlap S_in or M.
 * Supported: count <= 65535, dk <= 65535, dv <= 4096.
 */
kda_status kda_state_affine(const float *M, const float *B, const float *S_in,
                            float *S_out, int count, int dk, int dv, void *stream);

/*
 * kda_chunk_fwd_noalloc -- kda_chunk_fwd for callers that cannot allocate
 * device memory.  The paper has no counterpart: this is a deployment variant
 * of the bf16 chunked prefill.
 *
 * Who needs it: code running inside a host application that owns all device
 * memory and forbids its components from allocating (an inference engine that
 * reserves its whole budget up front, where an extra cudaMalloc fails or
 * breaks its accounting), and code on paths where an allocation call is not
 * permitted.  This entry point calls no cudaMalloc, cudaFree or other
 * allocating routine; its scratch is a fixed 32 MiB device array inside the
 * library, kept until the process exits.  The CUDA runtime reserves the array
 * on a device when it loads the library's module there: at load time, or,
 * under lazy module loading (CUDA_MODULE_LOADING=LAZY, the default since CUDA
 * 12.2), at this entry point's first call on the device.  A caller that
 * reserves its whole device budget up front should make one call (e.g. a
 * small warm-up) before it does.
 *
 * Arguments, layouts and results are those of kda_chunk_fwd.  Supported:
 * KDA_BF16 with dk = dv = 128 only (other dtypes/dims: KDA_ERR_UNSUPPORTED).
 * Size limit: it returns KDA_ERR_INVALID_ARG, with the needed and the
 * available byte counts in kda_last_error_message(), when
 *     roundup256(4 * (2 N + 1)) + slots * H * 74240 > 32 MiB,
 * where slots = B * ceil(T / 64) in dense mode and ceil(T / 64) + num_seqs in
 * varlen mode (e.g. 451 (chunk, head) slots: T = 1024 with H <= 28).
 * First call on a device: it looks up the array's device address there
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before any stream capture on the device.
 * Concurrency: every call uses the same array, which keeps the previous
 * call's contents (nothing in it needs to start cleared).  Calls whose work
 * overlaps on the GPU -- on different streams, or from different threads --
 * race on it; serialise them.
 */
kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v,
                                 const float *g, const float *beta,
                                 const float *initial_state, const int32_t *cu_seqlens,
                                 void *out, float *final_state,
                                 int B, int T, int H, int dk, int dv, int num_seqs,
                                 kda_dtype dtype, void *stream);

/*
 * kda_selftest_bounded_wait -- a diagnostic for the library's failure path.
 * The paper has no counterpart.
 *
 * Every kernel here that waits on an mbarrier polls it at most a bounded
 * number of times; when the bound runs out it sets the device error word to 1
 * (a wait timed out) and returns instead of hanging or trapping.  This call
 * launches one CTA that waits, polling at most `limit` times, on an mbarrier
 * nothing arrives on (no copy or MMA in flight), so it always times out: the
 * next kda_get_device_error() on the device reports code 1 and clears it, and
 * the context stays usable.  limit: 1 .. 65536 (else KDA_ERR_INVALID_ARG).
 */
kda_status kda_selftest_bounded_wait(unsigned limit, void *stream);

/* Static string for a status code. */
const char *kda_status_string(kda_status s);

/* Detail of the calling thread's last failing call ("" if none). */
const char *kda_last_error_message(void);

/*
 * Synchronises `stream`, then reads and clears the current device's error
 * word.  *code_out (may be NULL) receives the raw word (0 = clean).
 * Returns KDA_OK if the word was 0, KDA_ERR_DEVICE if it was set, or
 * KDA_ERR_CUDA if the synchronisation failed.
 */
kda_status kda_get_device_error(void *stream, int *code_out);

/* Library version, "major.minor.patch". */
const char *kda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KDA_B200_H */
