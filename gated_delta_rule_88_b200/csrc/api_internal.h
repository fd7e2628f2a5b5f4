// api_internal.h -- host-side helpers shared by the entry points of api.cu
// and noalloc.cu (argument checks, the bf16 prefill's scratch layout and
// launch sequence), so that the allocating and the allocation-free prefill
// cannot drift apart.
#pragma once
#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "common.cuh"
#include "kernels.h"

namespace kda {

// Detail of the calling thread's last failing call (kda_last_error_message).
extern thread_local char t_msg[512];

// Records the message for kda_last_error_message() and returns s.
kda_status fail(kda_status s, const char *fmt, ...);

// kda_chunk_fwd's argument rules (null pointers, sizes, dtype, varlen mode,
// alignment, problem size), with messages prefixed by fn.  On KDA_OK, *N_out
// is the number of sequences.  Enqueues nothing.
kda_status check_chunk_fwd_args(const char *fn, const void *q, const void *k, const void *v,
                                const float *g, const float *beta, const float *initial_state,
                                const int32_t *cu_seqlens, const void *out,
                                const float *final_state, int B, int T, int H, int dk, int dv,
                                int num_seqs, kda_dtype dtype, int *N_out);

// Scratch bytes of the bf16 (dk = dv = 128) prefill: the chunk offsets and
// the sequence order (256-byte rounded), then one record per (chunk slot,
// head).  *max_chunks (nullable)
// receives the chunk slots.
size_t bf16_prefill_scratch_bytes(int N, int B, int T, int H, bool varlen, long long *max_chunks);

// State-tile width (dv columns per chain CTA) for `units` (sequence, head)
// pairs on `sms` SMs.
int bf16_prefill_dvt(long long units, int sms);

// The bf16 prefill with no tokens: final = initial, or zeros.
cudaError_t bf16_prefill_no_tokens(const float *initial_state, float *final_state, int N, int H,
                                   cudaStream_t st);

// The bf16 prefill's launches (plan if varlen, prep, chain) on `scratch` of
// bf16_prefill_scratch_bytes() bytes.
cudaError_t launch_bf16_prefill(unsigned char *scratch, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *initial_state, const int32_t *cu_seqlens, void *out,
                                float *final_state, int B, int T, int H, int N, Prologue pro,
                                int sms, cudaStream_t st);

}  // namespace kda
