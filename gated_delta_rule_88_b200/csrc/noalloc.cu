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
// this module and stays allocated until the process exits.  The CUDA runtime
// reserves it when it loads the module on a device: at library load, or, with
// lazy module loading (CUDA_MODULE_LOADING=LAZY, the default since CUDA
// 12.2), at the first call of this entry point on that device.  A caller that
// reserves its whole device budget up front should make one call first.  Every call shares
// it; it keeps the last call's contents.  Nothing in it needs to start at
// zero: the plan and prep kernels write every byte the chain kernel later
// reads.  Two calls whose work overlaps on the GPU (e.g. on two streams, or
// two threads) race on the array and corrupt each other's results.
//
// The paper has no counterpart for this entry point; it is a deployment
// variant of the same kernels.
#include <mutex>

#include "../../include/kda.h"
#include "api_internal.h"
#include "common.cuh"

namespace {

constexpr size_t kStaticScratchBytes = 32u << 20;   // 32 MiB
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

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
    int N = 0;
    // the same argument rules as kda_chunk_fwd
    kda_status s = kda::check_chunk_fwd_args("kda_chunk_fwd_noalloc", q, k, v, g, beta,
                                             initial_state, cu_seqlens, out, final_state, B, T, H,
                                             dk, dv, num_seqs, dtype, &N);
    if (s != KDA_OK) return s;
    if (dtype != KDA_BF16 || dk != 128 || dv != 128)
        return kda::fail(KDA_ERR_UNSUPPORTED,
                         "kda_chunk_fwd_noalloc: only bf16 with dk = dv = 128 (got dtype %d, %d, %d)",
                         (int)dtype, dk, dv);
    long long max_chunks = 0;
    const size_t need = kda::bf16_prefill_scratch_bytes(N, B, T, H, cu_seqlens != nullptr, &max_chunks);
    if (need > kStaticScratchBytes)
        return kda::fail(KDA_ERR_INVALID_ARG,
                         "kda_chunk_fwd_noalloc: needs %zu bytes of scratch, the static maximum is %zu "
                         "(%lld chunk slots x %d heads; use kda_chunk_fwd)",
                         need, kStaticScratchBytes, max_chunks, H);
    cudaStream_t st = (cudaStream_t)stream;
    if (N == 0 || (long long)B * T == 0) {
        cudaError_t e = kda::bf16_prefill_no_tokens(initial_state, final_state, N, H, st);
        if (e != cudaSuccess)
            return kda::fail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc: %s", cudaGetErrorString(e));
        return KDA_OK;
    }
    unsigned char *scratch = nullptr;
    cudaError_t e = static_scratch(&scratch);
    if (e != cudaSuccess)
        return kda::fail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc: cudaGetSymbolAddress: %s",
                         cudaGetErrorString(e));
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    e = kda::launch_bf16_prefill(scratch, q, k, v, g, beta, initial_state, cu_seqlens, out,
                                 final_state, B, T, H, N, kda::Prologue{0, 1.f}, sms, st);
    if (e != cudaSuccess)
        return kda::fail(KDA_ERR_CUDA, "kda_chunk_fwd_noalloc launch: %s", cudaGetErrorString(e));
    return KDA_OK;
}

}  // extern "C"
