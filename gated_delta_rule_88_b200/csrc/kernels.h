// kernels.h -- internal launchers behind the C ABI (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Input prologue applied inside the kernels (the ABI's *_ex calls): bit 0
// L2-normalises q and k per (token, head), bit 1 takes sigmoid(beta); q is
// then multiplied by q_scale.  {0, 1.f} is the identity.
struct Prologue {
    int flags;
    float q_scale;
};

// Address of the current device's error word (see common.cuh), or nullptr.
int *error_word();

// One decode step for NH = N*H (sequence, head) pairs; state updated in place.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *out, int NH, int dk,
                          int dv, bool bf16, Prologue pro, cudaStream_t st);

// One decode token per sequence against a slot-indexed state pool
// [num_slots, H, dk, dv] (decode_step_kernel): sequence n uses entry slots[n]
// (n if null); a slot outside [0, num_slots) skips the sequence and sets the
// device error word.
cudaError_t launch_decode_slots(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *pool, const int32_t *slots,
                                int num_slots, void *out, int N, int H, int dk, int dv, bool bf16,
                                int *err, Prologue pro, cudaStream_t st);

// L decode tokens per sequence against a slot-indexed state pool
// [num_slots, H, dk, dv]; sequence n uses pool entry slots[n] (n if null).
// A persistent pipelined kernel (decode_pipe.cu): the next item's state
// arrives in shared memory while the current one is computed.  Per token the
// arithmetic is launch_decode's, operation for operation.
cudaError_t launch_decode_pipe(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *pool, const int32_t *slots, int num_slots,
                               void *out, int N, int H, int L, int dk, int dv, bool bf16, int *err,
                               Prologue pro, cudaStream_t st);

// The same call in the chunk form on tensor cores (decode_chunk.cu): bf16,
// dk = dv = 128, blocks of 16 tokens; bf16 operand rounding as in the prefill.
cudaError_t launch_decode_chunk(const void *q, const void *k, const void *v, const float *g,
                                const float *beta, float *pool, const int32_t *slots,
                                int num_slots, void *out, int N, int H, int L, int *err,
                                cudaStream_t st);
// The same, for listed (item, first token) pairs only; the count is read on
// the device.
cudaError_t launch_decode_chunk_list(const void *q, const void *k, const void *v, const float *g,
                                     const float *beta, float *pool, const int32_t *slots, int num_slots,
                                     void *out, int N, int H, int L, const int2 *list, const int *list_count,
                                     int *err, cudaStream_t st);
// The chunk-form decode on 64-token chunks on tcgen05 (decode_chunk_tc.cu),
// then the listed out-of-range items on the 16-token kernel.  `scratch`:
// decode_chunk_tc_scratch_bytes(N, H, sms) bytes, 256-byte aligned.
size_t decode_chunk_tc_scratch_bytes(int N, int H, int sms);
cudaError_t launch_decode_chunk_tc(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, float *pool, const int32_t *slots, int num_slots,
                                   void *out, int N, int H, int L, int sms, void *scratch, int *err,
                                   cudaStream_t st);

// Gradients of the recurrence (recurrent_bwd.cu): one warp per (sequence,
// head, 16-column state tile), workspace of recurrent_bwd_workspace bytes.
size_t recurrent_bwd_workspace(int B, int T, int H, int dk, int dv);
cudaError_t launch_recurrent_bwd(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *s0, const void *dout,
                                 const float *dsT, float *dq, float *dk, float *dv, float *dg,
                                 float *db, float *ds0, void *ws, int B, int T, int H, int dk_,
                                 int dv_, bool bf16, cudaStream_t st);

// Gated RMSNorm over rows of dv (64 or 128): y = x rsqrt(mean(x^2) + eps) w sigmoid(z).
cudaError_t launch_gated_rmsnorm(const void *x, const void *z, const float *w, float eps, void *y,
                                 long long rows, int dv, bool bf16, cudaStream_t st);

// S_out[i] = M[i] S_in[i] + B[i] (B may be null), i < count; M [count, dk, dk],
// B, S_in, S_out [count, dk, dv] fp32; S_out must not overlap S_in or M.
cudaError_t launch_state_affine(const float *M, const float *B, const float *S, float *out,
                                int count, int dk, int dv, cudaStream_t st);

// Exact-fp32 chunked prefill (SIMT).  dk, dv in {64, 128}.
// Token axis flattened: token t of the packed [B*T] axis, head h, channel c at
// ((t * H) + h) * d + c.  Sequences: dense (cu == nullptr, n-th spans
// [n*T, n*T+T)) or varlen (cu[n], cu[n+1]).
cudaError_t launch_chunk_f32(const void *q, const void *k, const void *v, const float *g,
                             const float *beta, const float *s0, const int32_t *cu,
                             void *out, float *sT, int N, int T, int total_T, int H,
                             int dk, int dv, bool bf16, Prologue pro, cudaStream_t st);

// bf16 tensor-core prefill (dk = dv = 128) in two launches over a scratch
// buffer of per-(chunk, head) records (chunk_ws.h):
//   chunk_plan  (varlen only) chunk offsets per sequence -> coff[N+1]
//   chunk_prep  parallel over (chunk, head): G, A, P, T, W, U, Qg, Kt, e^{G_C}
//               (A, P, W, U on tcgen05; err receives bounded-wait failures)
//   chunk_chain sequential over chunks per (sequence, head, dv tile),
//               tcgen05 MMAs with TMEM accumulators (chunk_chain_tc.cu)
size_t chunk_prep_smem_bytes();
// order (nullable): also the sequences sorted by decreasing length (ties by
// index; the identity order when N > 4096)
cudaError_t launch_chunk_plan(const int32_t *cu, int N, int total_T, int32_t *coff,
                              cudaStream_t st, int32_t *order = nullptr);
cudaError_t launch_chunk_prep(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, const int32_t *cu, const int32_t *coff,
                              int N, int T, int total_T, int H, int max_chunks,
                              unsigned char *wsp, Prologue pro, int *err, cudaStream_t st);
// s_img / v_img (nullable): per-(chunk, head) bf16 images of the state
// entering each chunk (32 KiB) and of V_new (16 KiB), for the backward.
// order (nullable): the sequences in launch order (longest first).
cudaError_t launch_chunk_chain(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
                               const float *s0, float *sT, void *out, int N, int T, int total_T,
                               int H, int dvt, int max_chunks, int *err, cudaStream_t st,
                               unsigned char *s_img = nullptr, unsigned char *v_img = nullptr,
                               const int32_t *order = nullptr);

// Chunked backward (bf16, dk = dv = 128): the reverse chain over the forward
// records (gradient images dS' 32 KiB and dV_new 16 KiB per (chunk, head)),
// then the per-(chunk, head) gradient pass.
cudaError_t launch_chunk_chain_bwd(const void *dout, const unsigned char *wsp, const int32_t *cu,
                                   const int32_t *coff, const float *dsT, float *ds0,
                                   unsigned char *dsp_img, unsigned char *dvn_img, int N, int T,
                                   int total_T, int H, int max_chunks, int *err, cudaStream_t st);
cudaError_t launch_chunk_bwd_local(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const void *dout, const int32_t *cu,
                                   const int32_t *coff, int N, int T, int total_T, int H,
                                   int max_chunks, const unsigned char *s_img,
                                   const unsigned char *v_img, const unsigned char *dsp_img,
                                   const unsigned char *dvn_img, float *dq, float *dk, float *dv,
                                   float *dg, float *dbeta, int *err, cudaStream_t st);

}  // namespace kda
