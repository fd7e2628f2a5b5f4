// api.cu -- the C ABI (include/kda.h): argument validation, dispatch,
// launch, status reporting.  All compute happens in the kernels this file
// launches; nothing here touches tensor data on the host.
#include <stdarg.h>
#include <stdio.h>

#include <mutex>

#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "common.cuh"
#include "kernels.h"
#include "chunk_ws.h"

namespace kda {
// The per-device error word (see common.cuh).  Host code reaches it through
// cudaMemcpy{To,From}Symbol, kernels through the address error_word() gives.
__device__ int g_device_error = 0;

int *error_word() {
    static int *addr[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = (int *)p;
    }
    return addr[dev];
}
}  // namespace kda

namespace kda {
// Detail of the calling thread's last failing call (kda_last_error_message).
thread_local char t_msg[512] = "";
}  // namespace kda

namespace {
using kda::t_msg;

kda_status fail(kda_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
    va_end(ap);
    return s;
}

kda_status cuda_fail(cudaError_t e, const char *what) {
    return fail(KDA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(e), cudaGetErrorName(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Library-private stream-ordered memory pool per device.  Its release
// threshold is unbounded, so scratch freed at the end of a call stays
// reserved for the next one instead of returning to the driver.
cudaError_t get_pool(cudaMemPool_t *out, int *sm_count) {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    static int sms[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!pools[dev]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = dev;
        cudaMemPool_t p;
        e = cudaMemPoolCreate(&p, &props);
        if (e != cudaSuccess) return e;
        uint64_t thr = ~0ull;
        e = cudaMemPoolSetAttribute(p, cudaMemPoolAttrReleaseThreshold, &thr);
        if (e != cudaSuccess) return e;
        e = cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        pools[dev] = p;
    }
    *out = pools[dev];
    *sm_count = sms[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_DEVICE: return "KDA_ERR_DEVICE";
    }
    return "KDA_ERR_UNKNOWN";
}

const char *kda_last_error_message(void) { return t_msg; }

const char *kda_version(void) { return "0.1.0"; }

kda_status kda_get_device_error(void *stream, int *code_out) {
    cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    int word = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&word, kda::g_device_error, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
    if (word != 0) {
        e = cudaMemcpyToSymbol(kda::g_device_error, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
    }
    if (code_out) *code_out = word;
    if (word != 0) return fail(KDA_ERR_DEVICE, "device error word = %d", word);
    return KDA_OK;
}

kda_status kda_recurrent_step(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state_inout, void *out, int N,
                              int H, int dk, int dv, kda_dtype dtype, void *stream) {
    t_msg[0] = 0;
    if (!q || !k || !v || !g || !beta || !state_inout || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_step: null pointer argument");
    if (N < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_step: bad sizes N=%d H=%d dk=%d dv=%d",
                    N, H, dk, dv);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_step: unknown dtype %d", (int)dtype);
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128)))
        return fail(KDA_ERR_UNSUPPORTED, "kda_recurrent_step: dk=%d dv=%d (supported: 64, 128)",
                    dk, dv);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) ||
        !aligned16(state_inout) || !aligned16(out))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_step: pointers must be 16-byte aligned");
    if ((uintptr_t)beta & 3u)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_step: beta must be 4-byte aligned");
    const long long NH = (long long)N * H;
    if (NH > 0x7fffffffLL)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_step: N*H too large");
    if (NH == 0) return KDA_OK;
    cudaError_t e = kda::launch_decode(q, k, v, g, beta, state_inout, out, (int)NH, dk, dv,
                                       dtype == KDA_BF16, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_step launch");
    return KDA_OK;
}

kda_status kda_recurrent_steps(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *state_pool, const int32_t *slots,
                               int num_slots, void *out, int N, int L, int H, int dk, int dv,
                               kda_dtype dtype, void *stream) {
    t_msg[0] = 0;
    if (!q || !k || !v || !g || !beta || !state_pool || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_steps: null pointer argument");
    if (N < 0 || L <= 0 || H <= 0 || dk <= 0 || dv <= 0 || num_slots <= 0)
        return fail(KDA_ERR_INVALID_ARG,
                    "kda_recurrent_steps: bad sizes N=%d L=%d H=%d dk=%d dv=%d num_slots=%d", N, L,
                    H, dk, dv, num_slots);
    if (!slots && num_slots < N)
        return fail(KDA_ERR_INVALID_ARG,
                    "kda_recurrent_steps: without slots the pool needs num_slots >= N (%d < %d)",
                    num_slots, N);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_steps: unknown dtype %d", (int)dtype);
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128)))
        return fail(KDA_ERR_UNSUPPORTED, "kda_recurrent_steps: dk=%d dv=%d (supported: 64, 128)",
                    dk, dv);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) ||
        !aligned16(state_pool) || !aligned16(out))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_steps: pointers must be 16-byte aligned");
    if (((uintptr_t)beta & 3u) || ((uintptr_t)slots & 3u))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_steps: beta and slots must be 4-byte aligned");
    const long long NH = (long long)N * H;
    if (NH > 0x7fffffffLL || (long long)N * L * H > (1LL << 40))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_steps: problem too large");
    if (NH == 0) return KDA_OK;
    cudaError_t e = kda::launch_decode_steps(q, k, v, g, beta, state_pool, slots, num_slots, out,
                                             N, H, L, dk, dv, dtype == KDA_BF16,
                                             kda::error_word(), (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_steps launch");
    return KDA_OK;
}

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *initial_state,
                         const int32_t *cu_seqlens, void *out, float *final_state, int B,
                         int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype,
                         void *stream) {
    t_msg[0] = 0;
    if (!q || !k || !v || !g || !beta || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: null pointer argument");
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: bad sizes B=%d T=%d H=%d dk=%d dv=%d",
                    B, T, H, dk, dv);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: unknown dtype %d", (int)dtype);
    int N = B;
    if (cu_seqlens) {
        if (B != 1)
            return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: varlen mode requires B == 1 (got %d)", B);
        if (num_seqs <= 0 || num_seqs > 65535)
            return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: num_seqs=%d out of [1, 65535]", num_seqs);
        N = num_seqs;
    } else if (B > 65535) {
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: B=%d exceeds 65535", B);
    }
    if (H > 65535) return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: H=%d exceeds 65535", H);
    const void *ptrs[] = {q, k, v, g, out, initial_state, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: pointers must be 16-byte aligned");
    if (((uintptr_t)beta & 3u) || (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: beta and cu_seqlens must be 4-byte aligned");
    const long long total_T = (long long)B * T;
    if (total_T > 0x7fffffffLL || total_T * H > (1LL << 40))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd: problem too large (B*T=%lld)", total_T);
    cudaStream_t st = (cudaStream_t)stream;

    if (dtype == KDA_F32) {
        if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128)))
            return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd(f32): dk=%d dv=%d (supported: 64, 128)",
                        dk, dv);
        cudaError_t e = kda::launch_chunk_f32(
            (const float *)q, (const float *)k, (const float *)v, g, beta, initial_state,
            cu_seqlens, (float *)out, final_state, N, T, (int)total_T, H, dk, dv, st);
        if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(f32) launch");
        return KDA_OK;
    }
    if (dk != 128 || dv != 128)
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd(bf16): dk=%d dv=%d (supported: 128, 128)",
                    dk, dv);
    if (N == 0 || total_T == 0) {
        // nothing to process: final = initial (or zeros)
        if (final_state) {
            const size_t bytes = (size_t)N * H * dk * dv * sizeof(float);
            cudaError_t e = initial_state
                ? (initial_state == final_state ? cudaSuccess
                   : cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, st))
                : cudaMemsetAsync(final_state, 0, bytes, st);
            if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) empty input");
        }
        return KDA_OK;
    }
    const long long max_chunks = cu_seqlens ? (total_T + 63) / 64 + N : (long long)B * ((T + 63) / 64);
    const size_t coff_bytes = (((size_t)N + 1) * sizeof(int32_t) + 255) & ~(size_t)255;
    const size_t bytes = coff_bytes + (size_t)max_chunks * H * kda::ws::RECORD;
    cudaMemPool_t pool;
    int sms = 148;
    cudaError_t e = get_pool(&pool, &sms);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) memory pool");
    void *scratch = nullptr;
    e = cudaMallocFromPoolAsync(&scratch, bytes, pool, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) scratch allocation");
    int32_t *coff = (int32_t *)scratch;
    unsigned char *records = (unsigned char *)scratch + coff_bytes;
    const long long units = (long long)N * H;
    const int dvt = units * 8 <= sms ? 16 : units * 4 <= sms ? 32 : 64;
    if (cu_seqlens) e = kda::launch_chunk_plan(cu_seqlens, N, (int)total_T, coff, st);
    if (e == cudaSuccess)
        e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, coff, N, T, (int)total_T, H,
                                   (int)max_chunks, records, st);
    if (e == cudaSuccess)
        e = kda::launch_chunk_chain(records, cu_seqlens, coff, initial_state, final_state, out, N,
                                    T, (int)total_T, H, dvt, (int)max_chunks, kda::error_word(), st);
    cudaError_t e2 = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) launch");
    if (e2 != cudaSuccess) return cuda_fail(e2, "kda_chunk_fwd(bf16) scratch release");
    return KDA_OK;
}

}  // extern "C"
