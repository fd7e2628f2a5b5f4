// kernels.h -- internal launchers behind the C ABI (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// One decode step for NH = N*H (sequence, head) pairs; state updated in place.
cudaError_t launch_decode(const void *q, const void *k, const void *v, const float *g,
                          const float *beta, float *state, void *out, int NH, int dk,
                          int dv, bool bf16, cudaStream_t st);

// Exact-fp32 chunked prefill (SIMT).  dk, dv in {64, 128}.
// Token axis flattened: token t of the packed [B*T] axis, head h, channel c at
// ((t * H) + h) * d + c.  Sequences: dense (cu == nullptr, n-th spans
// [n*T, n*T+T)) or varlen (cu[n], cu[n+1]).
cudaError_t launch_chunk_f32(const float *q, const float *k, const float *v, const float *g,
                             const float *beta, const float *s0, const int32_t *cu,
                             float *out, float *sT, int N, int T, int total_T, int H,
                             int dk, int dv, cudaStream_t st);

}  // namespace kda
