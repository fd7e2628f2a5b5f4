// noalloc.cu -- kda_chunk_fwd_noalloc: the bf16 chunked prefill without any
// device allocation, for callers that cannot allocate.
//
// Who needs it: code embedded in a host process that owns all device memory
// and forbids its plugins from allocating (an inference engine that reserves
// its whole memory budget up front, so any extra cudaMalloc fails or breaks
// its accounting), and code on paths where an allocation call is not allowed
// or would stall the device.  kda_chunk_fwd takes its scratch from a
// stream-ordered pool; this variant uses a fixed, file-scope device array
// instead and calls no cudaMalloc, cudaFree or any allocating routine.
//
// The array (kStaticScratchBytes, 32 MiB) exists once per device that loads
// the library and stays allocated until the process exits.  Every call shares
// it; it keeps the last call's contents.  Nothing in it needs to start at
// zero: the plan and prep kernels write every byte the chain kernel later
// reads.  Two calls whose work overlaps on the GPU (e.g. on two streams, or
// two threads) race on the array and corrupt each other's results.
//
// The paper has no counterpart for this entry point; it is a deployment
// variant of the same kernels.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include "../../include/kda.h"
#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"

namespace kda {
extern thread_local char t_msg[512];
}

namespace {

constexpr size_t kStaticScratchBytes = 32u << 20;   // 32 MiB
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Failures are described through kda_last_error_message(), like every entry point.
kda_status nfail(kda_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(kda::t_msg, sizeof(kda::t_msg), fmt, ap);
    va_end(ap);
    return s;
}

// Device address of g_static_scratch on the current device.  In host code the
// array's name is only a host-side stand-in; the address must come from
// cudaGetSymbolAddress with the device current.  Looked up once per device.
cudaError_t static_scratch(unsigned char **out) {
    static std::mutex mu;
    static unsigned char *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return e;
        addr[dev] = (unsigned char *)p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

kda_status kda_chunk_fwd_noalloc(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *initial_state,
                                 const int32_t *cu_seqlens, void *out, float *final_state,
                                 int B, int T, int H, int dk, int dv, int num_seqs,
                                 kda_dtype dtype, void *stream) {
    kda::t_msg[0] = 0;
    if (!q || !k || !v || !g || !beta || !out)
        return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: null pointer argument");
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: bad sizes B=%d T=%d H=%d dk=%d dv=%d",
                     B, T, H, dk, dv);
    if (dtype != KDA_BF16 || dk != 128 || dv != 128)
        return nfail(KDA_ERR_UNSUPPORTED,
                     "kda_chunk_fwd_noalloc: only bf16 with dk = dv = 128 (got dtype %d, %d, %d)",
                     (int)dtype, dk, dv);
    int N = B;
    if (cu_seqlens) {
        if (B != 1)
            return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: varlen mode requires B == 1");
        if (num_seqs <= 0 || num_seqs > 65535)
            return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: num_seqs=%d out of [1, 65535]",
                         num_seqs);
        N = num_seqs;
    } else if (B > 65535) {
        return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: B=%d exceeds 65535", B);
    }
    if (H > 65535) return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: H=%d exceeds 65535", H);
    const void *ptrs[] = {q, k, v, g, out, initial_state, final_state};
    for (const void *p : ptrs)
        if (p && ((uintptr_t)p & 15u))
            return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: pointers must be 16-byte aligned");
    if (((uintptr_t)beta & 3u) || (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)))
        return nfail(KDA_ERR_INVALID_ARG,
                     "kda_chunk_fwd_noalloc: beta and cu_seqlens must be 4-byte aligned");
    const long long total_T = (long long)B * T;
    if (total_T > 0x7fffffffLL)
        return nfail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_noalloc: problem too large (B*T=%lld)", total_T);
    const long long max_chunks = cu_seqlens ? (total_T + 63) / 64 + N : (long long)B * ((T + 63) / 64);
    const size_t coff_bytes = (((size_t)N + 1) * sizeof(int32_t) + 255) & ~(size_t)255;
    const size_t need = coff_bytes + (size_t)max_chunks * H * kda::ws::RECORD;
    if (need > kStaticScratchBytes)
        return nfail(KDA_ERR_INVALID_ARG,
                     "kda_chunk_fwd_noalloc: needs %zu bytes of scratch, the static maximum is %zu "
                     "(%lld chunk slots x %d heads; use kda_chunk_fwd)",
                     need, kStaticScratchBytes, max_chunks, H);
    cudaStream_t st = (cudaStream_t)stream;
    if (N == 0 || total_T == 0) {
        if (final_state) {
            const size_t bytes = (size_t)N * H * dk * dv * sizeof(float);
            cudaError_t e = initial_state
                ? (initial_state == final_state ? cudaSuccess
                   : cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, st))
                : cudaMemsetAsync(final_state, 0, bytes, st);
            if (e != cudaSuccess)
                return nfail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc: %s", cudaGetErrorString(e));
        }
        return KDA_OK;
    }
    unsigned char *scratch = nullptr;
    cudaError_t e = static_scratch(&scratch);
    if (e != cudaSuccess)
        return nfail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc: cudaGetSymbolAddress: %s",
                     cudaGetErrorString(e));
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int32_t *coff = (int32_t *)scratch;
    unsigned char *records = scratch + coff_bytes;
    const long long units = (long long)N * H;
    const int dvt = units * 8 <= sms ? 16 : units * 4 <= sms ? 32 : 64;
    if (cu_seqlens) e = kda::launch_chunk_plan(cu_seqlens, N, (int)total_T, coff, st);
    if (e == cudaSuccess)
        e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, coff, N, T, (int)total_T, H,
                                   (int)max_chunks, records, kda::Prologue{0, 1.f}, kda::error_word(), st);
    if (e == cudaSuccess)
        e = kda::launch_chunk_chain(records, cu_seqlens, coff, initial_state, final_state, out, N,
                                    T, (int)total_T, H, dvt, (int)max_chunks, kda::error_word(), st);
    if (e != cudaSuccess)
        return nfail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc launch: %s", cudaGetErrorString(e));
    return KDA_OK;
}

}  // extern "C"
