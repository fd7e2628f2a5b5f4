// api.cu -- the C ABI (include/kda.h): argument validation, dispatch,
// launch, status reporting.  All compute happens in the kernels this file
// launches; nothing here touches tensor data on the host.
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/kda.h"
#include "common.cuh"
#include "kernels.h"

// Chunk-form serving decode: from this many tokens per call on, 64-token
// chunks on tcgen05 (decode_chunk_tc.cu); below it, 16-token blocks
// (decode_chunk.cu).
#ifndef KDA_TC_CHUNK_MIN_L
#define KDA_TC_CHUNK_MIN_L 33
#endif
#include "chunk_ws.h"
#include "api_internal.h"

namespace kda {
// The per-device error word (see common.cuh).  Host code reaches it through
// cudaMemcpy{To,From}Symbol, kernels through the address error_word() gives.
__device__ int g_device_error = 0;

int *error_word() {
    // per-device cache; threads that race on first use store the same address
    static std::atomic<int *> addr[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    int *p = addr[dev].load(std::memory_order_acquire);
    if (!p) {
        void *s = nullptr;
        if (cudaGetSymbolAddress(&s, g_device_error) != cudaSuccess) return nullptr;
        p = (int *)s;
        addr[dev].store(p, std::memory_order_release);
    }
    return p;
}
}  // namespace kda

namespace kda {
// Detail of the calling thread's last failing call (kda_last_error_message).
thread_local char t_msg[512] = "";
}  // namespace kda

namespace kda {
kda_status fail(kda_status s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
    va_end(ap);
    return s;
}
}  // namespace kda

namespace {
using kda::t_msg;
using kda::fail;

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

static kda_status chunk_fwd_device(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *initial_state,
                                   const int32_t *cu_seqlens, void *out, float *final_state,
                                   int B, int T, int H, int dk, int dv, int N, kda_dtype dtype,
                                   kda::Prologue pro, cudaStream_t st);

// flags of the *_ex calls -> kernel prologue
static kda_status make_prologue(const char *fn, unsigned flags, float q_scale,
                                kda::Prologue *pro) {
    if (flags & ~(unsigned)(KDA_QK_L2NORM | KDA_BETA_SIGMOID))
        return fail(KDA_ERR_INVALID_ARG, "%s: unknown flag bits 0x%x", fn, flags);
    if (!(q_scale == q_scale) || q_scale > 3.4e38f || q_scale < -3.4e38f)
        return fail(KDA_ERR_INVALID_ARG, "%s: q_scale must be finite", fn);
    pro->flags = (flags & KDA_QK_L2NORM ? kda::kProQkL2Norm : 0) |
                 (flags & KDA_BETA_SIGMOID ? kda::kProBetaSigmoid : 0);
    pro->q_scale = q_scale;
    return KDA_OK;
}

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

static kda_status recurrent_step_impl(const void *q, const void *k, const void *v,
                                      const float *g, const float *beta, float *state_inout,
                                      void *out, int N, int H, int dk, int dv, kda_dtype dtype,
                                      kda::Prologue pro, void *stream) {
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
                                       dtype == KDA_BF16, pro, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_step launch");
    return KDA_OK;
}

kda_status kda_recurrent_step(const void *q, const void *k, const void *v, const float *g,
                              const float *beta, float *state_inout, void *out, int N,
                              int H, int dk, int dv, kda_dtype dtype, void *stream) {
    t_msg[0] = 0;
    return recurrent_step_impl(q, k, v, g, beta, state_inout, out, N, H, dk, dv, dtype,
                               kda::Prologue{0, 1.f}, stream);
}

kda_status kda_recurrent_step_ex(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, float *state_inout, void *out, int N,
                                 int H, int dk, int dv, kda_dtype dtype, unsigned flags,
                                 float q_scale, void *stream) {
    t_msg[0] = 0;
    kda::Prologue pro;
    kda_status st = make_prologue("kda_recurrent_step_ex", flags, q_scale, &pro);
    if (st != KDA_OK) return st;
    return recurrent_step_impl(q, k, v, g, beta, state_inout, out, N, H, dk, dv, dtype, pro,
                               stream);
}

kda_status kda_recurrent_steps(const void *q, const void *k, const void *v, const float *g,
                               const float *beta, float *state_pool, const int32_t *slots,
                               int num_slots, void *out, int N, int L, int H, int dk, int dv,
                               kda_dtype dtype, unsigned flags, float q_scale, void *stream) {
    t_msg[0] = 0;
    kda::Prologue pro;
    const bool chunk = (flags & KDA_STEPS_CHUNK) != 0;
    kda_status pst = make_prologue("kda_recurrent_steps", flags & ~(unsigned)KDA_STEPS_CHUNK,
                                   q_scale, &pro);
    if (pst != KDA_OK) return pst;
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
    const bool tc = chunk && L >= 2 && dtype == KDA_BF16 && dk == 128 && dv == 128 &&
                    pro.flags == 0 && pro.q_scale == 1.f;
    cudaStream_t st = (cudaStream_t)stream;
    // (the 64-token path moves the state and the output in 32-byte pieces)
    if (tc && L >= KDA_TC_CHUNK_MIN_L && !((uintptr_t)state_pool & 31u) && !((uintptr_t)out & 31u)) {
        // 64-token chunks on tcgen05, with a scratch of per-CTA slots and
        // the list of out-of-range items
        cudaMemPool_t mp;
        int sms = 148;
        cudaError_t e = get_pool(&mp, &sms);
        if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_steps memory pool");
        void *scratch = nullptr;
        e = cudaMallocFromPoolAsync(&scratch, kda::decode_chunk_tc_scratch_bytes(N, H, sms), mp, st);
        if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_steps scratch allocation");
        e = kda::launch_decode_chunk_tc(q, k, v, g, beta, state_pool, slots, num_slots, out, N, H, L, sms,
                                        scratch, kda::error_word(), st);
        cudaError_t e2 = cudaFreeAsync(scratch, st);
        if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_steps launch");
        if (e2 != cudaSuccess) return cuda_fail(e2, "kda_recurrent_steps scratch release");
        return KDA_OK;
    }
    cudaError_t e = tc ? kda::launch_decode_chunk(q, k, v, g, beta, state_pool, slots, num_slots,
                                                  out, N, H, L, kda::error_word(), st)
                       : kda::launch_decode_pipe(q, k, v, g, beta, state_pool, slots, num_slots, out,
                                                 N, H, L, dk, dv, dtype == KDA_BF16,
                                                 kda::error_word(), pro, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_steps launch");
    return KDA_OK;
}

static kda_status chunk_fwd_impl(const void *q, const void *k, const void *v, const float *g,
                                 const float *beta, const float *initial_state,
                                 const int32_t *cu_seqlens, void *out, float *final_state,
                                 int B, int T, int H, int dk, int dv, int num_seqs,
                                 kda_dtype dtype, kda::Prologue pro, void *stream) {
    int N = 0;
    kda_status s = kda::check_chunk_fwd_args("kda_chunk_fwd", q, k, v, g, beta, initial_state,
                                             cu_seqlens, out, final_state, B, T, H, dk, dv,
                                             num_seqs, dtype, &N);
    if (s != KDA_OK) return s;
    return chunk_fwd_device(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, B, T,
                            H, dk, dv, N, dtype, pro, (cudaStream_t)stream);
}

kda_status kda_chunk_fwd(const void *q, const void *k, const void *v, const float *g,
                         const float *beta, const float *initial_state,
                         const int32_t *cu_seqlens, void *out, float *final_state, int B,
                         int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype,
                         void *stream) {
    t_msg[0] = 0;
    return chunk_fwd_impl(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, B, T,
                          H, dk, dv, num_seqs, dtype, kda::Prologue{0, 1.f}, stream);
}

kda_status kda_chunk_fwd_ex(const void *q, const void *k, const void *v, const float *g,
                            const float *beta, const float *initial_state,
                            const int32_t *cu_seqlens, void *out, float *final_state, int B,
                            int T, int H, int dk, int dv, int num_seqs, kda_dtype dtype,
                            unsigned flags, float q_scale, void *stream) {
    t_msg[0] = 0;
    kda::Prologue pro;
    kda_status st = make_prologue("kda_chunk_fwd_ex", flags, q_scale, &pro);
    if (st != KDA_OK) return st;
    return chunk_fwd_impl(q, k, v, g, beta, initial_state, cu_seqlens, out, final_state, B, T,
                          H, dk, dv, num_seqs, dtype, pro, stream);
}

}  // extern "C"

namespace kda {

kda_status check_chunk_fwd_args(const char *fn, const void *q, const void *k, const void *v,
                                const float *g, const float *beta, const float *initial_state,
                                const int32_t *cu_seqlens, const void *out,
                                const float *final_state, int B, int T, int H, int dk, int dv,
                                int num_seqs, kda_dtype dtype, int *N_out) {
    if (!q || !k || !v || !g || !beta || !out)
        return fail(KDA_ERR_INVALID_ARG, "%s: null pointer argument", fn);
    if (B <= 0 || T < 0 || H <= 0 || dk <= 0 || dv <= 0)
        return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes B=%d T=%d H=%d dk=%d dv=%d", fn, B, T, H,
                    dk, dv);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
    int N = B;
    if (cu_seqlens) {
        if (B != 1)
            return fail(KDA_ERR_INVALID_ARG, "%s: varlen mode requires B == 1 (got %d)", fn, B);
        if (num_seqs <= 0 || num_seqs > 65535)
            return fail(KDA_ERR_INVALID_ARG, "%s: num_seqs=%d out of [1, 65535]", fn, num_seqs);
        N = num_seqs;
    } else if (B > 65535) {
        return fail(KDA_ERR_INVALID_ARG, "%s: B=%d exceeds 65535", fn, B);
    }
    if (H > 65535) return fail(KDA_ERR_INVALID_ARG, "%s: H=%d exceeds 65535", fn, H);
    const void *ptrs[] = {q, k, v, g, out, initial_state, final_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(KDA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    if (((uintptr_t)beta & 3u) || (cu_seqlens && ((uintptr_t)cu_seqlens & 3u)))
        return fail(KDA_ERR_INVALID_ARG, "%s: beta and cu_seqlens must be 4-byte aligned", fn);
    const long long total_T = (long long)B * T;
    if (total_T > 0x7fffffffLL || total_T * H > (1LL << 40))
        return fail(KDA_ERR_INVALID_ARG, "%s: problem too large (B*T=%lld)", fn, total_T);
    *N_out = N;
    return KDA_OK;
}

// chunk offsets coff[N + 1], then (varlen) the sequence order[N], 256-byte rounded
static size_t plan_bytes(int N) { return (((size_t)2 * N + 1) * sizeof(int32_t) + 255) & ~(size_t)255; }

size_t bf16_prefill_scratch_bytes(int N, int B, int T, int H, bool varlen, long long *max_chunks) {
    const long long total_T = (long long)B * T;
    const long long mc = varlen ? (total_T + 63) / 64 + N : (long long)B * ((T + 63) / 64);
    if (max_chunks) *max_chunks = mc;
    return plan_bytes(N) + (size_t)mc * H * ws::RECORD;
}

cudaError_t bf16_prefill_no_tokens(const float *initial_state, float *final_state, int N, int H,
                                   cudaStream_t st) {
    // nothing to process: final = initial (or zeros)
    if (!final_state) return cudaSuccess;
    const size_t bytes = (size_t)N * H * 128 * 128 * sizeof(float);
    if (!initial_state) return cudaMemsetAsync(final_state, 0, bytes, st);
    if (initial_state == final_state) return cudaSuccess;
    return cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice, st);
}

int bf16_prefill_dvt(long long units, int sms) {
    // the widest state tile that still gives every SM a chain: one CTA per
    // (sequence, head) once there are more of those than half the SMs
    return units * 8 <= sms ? 16 : units * 4 <= sms ? 32 : units * 2 <= sms ? 64 : 128;
}

cudaError_t launch_bf16_prefill(unsigned char *scratch, const void *q, const void *k,
                                const void *v, const float *g, const float *beta,
                                const float *initial_state, const int32_t *cu_seqlens, void *out,
                                float *final_state, int B, int T, int H, int N, Prologue pro,
                                int sms, cudaStream_t st) {
    const long long total_T = (long long)B * T;
    long long max_chunks = 0;
    bf16_prefill_scratch_bytes(N, B, T, H, cu_seqlens != nullptr, &max_chunks);
    int32_t *coff = (int32_t *)scratch;
    int32_t *order = cu_seqlens ? coff + N + 1 : nullptr;
    unsigned char *records = scratch + plan_bytes(N);
    const int dvt = bf16_prefill_dvt((long long)N * H, sms);
    cudaError_t e = cudaSuccess;
    if (cu_seqlens) e = launch_chunk_plan(cu_seqlens, N, (int)total_T, coff, st, order);
    if (e == cudaSuccess)
        e = launch_chunk_prep(q, k, v, g, beta, cu_seqlens, coff, N, T, (int)total_T, H,
                              (int)max_chunks, records, pro, error_word(), st);
    if (e == cudaSuccess)
        e = launch_chunk_chain(records, cu_seqlens, coff, initial_state, final_state, out, N, T,
                               (int)total_T, H, dvt, (int)max_chunks, error_word(), st, nullptr,
                               nullptr, order);
    return e;
}

}  // namespace kda

// Device-side part of kda_chunk_fwd (arguments already validated).
static kda_status chunk_fwd_device(const void *q, const void *k, const void *v, const float *g,
                                   const float *beta, const float *initial_state,
                                   const int32_t *cu_seqlens, void *out, float *final_state,
                                   int B, int T, int H, int dk, int dv, int N, kda_dtype dtype,
                                   kda::Prologue pro, cudaStream_t st) {
    const long long total_T = (long long)B * T;
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128)))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd: dk=%d dv=%d (supported: 64, 128)", dk, dv);
    if (dtype == KDA_F32 || dk != 128 || dv != 128) {
        // fp32 arithmetic on the CUDA cores: fp32 inputs, and bf16 inputs at
        // head dimensions the tensor-core kernels do not take
        cudaError_t e = kda::launch_chunk_f32(q, k, v, g, beta, initial_state, cu_seqlens, out,
                                              final_state, N, T, (int)total_T, H, dk, dv,
                                              dtype == KDA_BF16, pro, st);
        if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(simt) launch");
        return KDA_OK;
    }
    if (N == 0 || total_T == 0) {
        cudaError_t e = kda::bf16_prefill_no_tokens(initial_state, final_state, N, H, st);
        if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) empty input");
        return KDA_OK;
    }
    const size_t bytes = kda::bf16_prefill_scratch_bytes(N, B, T, H, cu_seqlens != nullptr, nullptr);
    cudaMemPool_t pool;
    int sms = 148;
    cudaError_t e = get_pool(&pool, &sms);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) memory pool");
    void *scratch = nullptr;
    e = cudaMallocFromPoolAsync(&scratch, bytes, pool, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) scratch allocation");
    e = kda::launch_bf16_prefill((unsigned char *)scratch, q, k, v, g, beta, initial_state,
                                 cu_seqlens, out, final_state, B, T, H, N, pro, sms, st);
    cudaError_t e2 = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd(bf16) launch");
    if (e2 != cudaSuccess) return cuda_fail(e2, "kda_chunk_fwd(bf16) scratch release");
    return KDA_OK;
}

extern "C" kda_status kda_gated_rmsnorm(const void *x, const void *gate, const float *weight,
                                        float eps, void *out, long long rows, int dv,
                                        kda_dtype dtype, void *stream) {
    t_msg[0] = 0;
    if (!x || !gate || !weight || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_gated_rmsnorm: null pointer argument");
    if (rows < 0 || rows > (1LL << 36))
        return fail(KDA_ERR_INVALID_ARG, "kda_gated_rmsnorm: bad row count %lld", rows);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "kda_gated_rmsnorm: unknown dtype %d", (int)dtype);
    if (!(eps >= 0.f) || eps > 3.4e38f)
        return fail(KDA_ERR_INVALID_ARG, "kda_gated_rmsnorm: eps must be finite and >= 0");
    if (dv != 64 && dv != 128)
        return fail(KDA_ERR_UNSUPPORTED, "kda_gated_rmsnorm: dv=%d (supported: 64, 128)", dv);
    if (!aligned16(x) || !aligned16(gate) || !aligned16(out) || ((uintptr_t)weight & 3u))
        return fail(KDA_ERR_INVALID_ARG,
                    "kda_gated_rmsnorm: x, gate, out must be 16-byte aligned, weight 4-byte");
    cudaError_t e = kda::launch_gated_rmsnorm(x, gate, weight, eps, out, rows, dv, dtype == KDA_BF16,
                                              (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kda_gated_rmsnorm launch");
    return KDA_OK;
}

// Saved forward intermediates for the chunked backward (kda_chunk_fwd_save):
// the plan (chunk offsets and sequence order), then per (chunk slot, head)
// the record (74,240 B), then the bf16 images of the state entering each
// chunk (32 KiB) and of V_new (16 KiB).
namespace {
struct SavedLayout {
    long long max_chunks = 0;
    size_t plan = 0, records = 0, s_img = 0, v_img = 0, total = 0;
};
SavedLayout saved_layout(int N, int B, int T, int H, bool varlen) {
    SavedLayout L;
    const long long total_T = (long long)B * T;
    L.max_chunks = varlen ? (total_T + 63) / 64 + N : (long long)B * ((T + 63) / 64);
    const size_t slots = (size_t)L.max_chunks * H;
    L.plan = 0;
    L.records = (((size_t)2 * N + 1) * sizeof(int32_t) + 255) & ~(size_t)255;
    L.s_img = L.records + slots * kda::ws::RECORD;
    L.v_img = L.s_img + slots * 32768;
    L.total = L.v_img + slots * 16384;
    return L;
}

// Argument rules shared by kda_chunk_bwd and kda_chunk_bwd_saved.
kda_status check_chunk_bwd_args(const char *fn, const void *q, const void *k, const void *v,
                                const float *g, const float *beta, const float *initial_state,
                                const int32_t *cu_seqlens, const void *dout,
                                const float *dfinal_state, const float *dq, const float *dk,
                                const float *dv, const float *dg, const float *dbeta,
                                const float *dinitial_state, int B, int T, int H, int dk_,
                                int dv_, int num_seqs, kda_dtype dtype, int *N_out) {
    if (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta)
        return fail(KDA_ERR_INVALID_ARG, "%s: null pointer argument", fn);
    if (B <= 0 || T < 0 || H <= 0 || dk_ <= 0 || dv_ <= 0 || B > 65535 || H > 65535)
        return fail(KDA_ERR_INVALID_ARG, "%s: bad sizes B=%d T=%d H=%d dk=%d dv=%d", fn, B, T, H,
                    dk_, dv_);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "%s: unknown dtype %d", fn, (int)dtype);
    if (dtype != KDA_BF16 || dk_ != 128 || dv_ != 128)
        return fail(KDA_ERR_UNSUPPORTED,
                    "%s: dtype=%d dk=%d dv=%d (supported: bf16 with dk = dv = 128)", fn,
                    (int)dtype, dk_, dv_);
    int N = B;
    if (cu_seqlens) {
        if (B != 1)
            return fail(KDA_ERR_INVALID_ARG, "%s: varlen mode requires B == 1 (got %d)", fn, B);
        if (num_seqs <= 0 || num_seqs > 65535)
            return fail(KDA_ERR_INVALID_ARG, "%s: num_seqs=%d out of [1, 65535]", fn, num_seqs);
        N = num_seqs;
    }
    const void *ptrs[] = {q, k, v, g, dout, dq, dk, dv, dg, initial_state, dfinal_state, dinitial_state};
    for (const void *p : ptrs)
        if (p && !aligned16(p))
            return fail(KDA_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
    if (((uintptr_t)beta & 3u) || ((uintptr_t)dbeta & 3u) || ((uintptr_t)cu_seqlens & 3u))
        return fail(KDA_ERR_INVALID_ARG, "%s: beta, dbeta and cu_seqlens must be 4-byte aligned", fn);
    const long long total_T = (long long)B * T;
    if (total_T > 0x7fffffffLL || total_T * H > (1LL << 34))
        return fail(KDA_ERR_INVALID_ARG, "%s: problem too large (B*T=%lld)", fn, total_T);
    *N_out = N;
    return KDA_OK;
}

// The backward's launches; saved (nullable) holds the forward's plan,
// records and images (kda_chunk_fwd_save), else they are recomputed.
kda_status chunk_bwd_run(const char *fn, const void *q, const void *k, const void *v,
                         const float *g, const float *beta, const float *initial_state,
                         const int32_t *cu_seqlens, const void *dout, const float *dfinal_state,
                         float *dq, float *dk, float *dv, float *dg, float *dbeta,
                         float *dinitial_state, int B, int T, int H, int N,
                         const unsigned char *saved, cudaStream_t st) {
    const long long total_T = (long long)B * T;
    const size_t sbytes = (size_t)N * H * 128 * 128 * sizeof(float);
    if (total_T == 0) {
        // no tokens: the initial state's gradient is the final state's
        cudaError_t e = cudaSuccess;
        if (dinitial_state)
            e = dfinal_state ? cudaMemcpyAsync(dinitial_state, dfinal_state, sbytes,
                                               cudaMemcpyDeviceToDevice, st)
                             : cudaMemsetAsync(dinitial_state, 0, sbytes, st);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, fn);
    }
    const SavedLayout L = saved_layout(N, B, T, H, cu_seqlens != nullptr);
    const size_t slots = (size_t)L.max_chunks * H;
    // scratch: the gradient images, and (recompute) a copy of the saved layout
    const size_t bytes = slots * (32768 + 16384) + (saved ? 0 : L.total);
    cudaMemPool_t pool;
    int sms = 148;
    cudaError_t e = get_pool(&pool, &sms);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    void *scratch = nullptr;
    e = cudaMallocFromPoolAsync(&scratch, bytes, pool, st);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    unsigned char *dsp_img = (unsigned char *)scratch;
    unsigned char *dvn_img = dsp_img + slots * 32768;
    unsigned char *fwd = saved ? nullptr : dvn_img + slots * 16384;
    const unsigned char *base = saved ? saved : fwd;
    const int32_t *coff = (const int32_t *)(base + L.plan);
    const unsigned char *records = base + L.records;
    const unsigned char *s_img = base + L.s_img, *v_img = base + L.v_img;
    int *err = kda::error_word();
    if (!saved) {
        // forward recompute: plan, records, then the chain storing S and V_new per chunk
        kda::Prologue pro{0, 1.f};
        if (cu_seqlens) e = kda::launch_chunk_plan(cu_seqlens, N, (int)total_T, (int32_t *)coff, st);
        if (e == cudaSuccess)
            e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, cu_seqlens ? coff : nullptr, N,
                                       T, (int)total_T, H, (int)L.max_chunks,
                                       fwd + L.records, pro, err, st);
        if (e == cudaSuccess)
            e = kda::launch_chunk_chain(records, cu_seqlens, cu_seqlens ? coff : nullptr,
                                        initial_state, nullptr, nullptr, N, T, (int)total_T, H, 32,
                                        (int)L.max_chunks, err, st, fwd + L.s_img, fwd + L.v_img);
    }
    // reverse chain, then the per-(chunk, head) gradients
    if (e == cudaSuccess)
        e = kda::launch_chunk_chain_bwd(dout, records, cu_seqlens, cu_seqlens ? coff : nullptr,
                                        dfinal_state, dinitial_state, dsp_img, dvn_img, N, T,
                                        (int)total_T, H, (int)L.max_chunks, err, st);
    if (e == cudaSuccess)
        e = kda::launch_chunk_bwd_local(q, k, v, g, beta, dout, cu_seqlens,
                                        cu_seqlens ? coff : nullptr, N, T, (int)total_T, H,
                                        (int)L.max_chunks, s_img, v_img, dsp_img, dvn_img, dq, dk,
                                        dv, dg, dbeta, err, st);
    cudaError_t e2 = cudaFreeAsync(scratch, st);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    if (e2 != cudaSuccess) return cuda_fail(e2, fn);
    return KDA_OK;
}
}  // namespace

extern "C" kda_status kda_chunk_bwd(const void *q, const void *k, const void *v, const float *g,
                                    const float *beta, const float *initial_state,
                                    const int32_t *cu_seqlens, const void *dout,
                                    const float *dfinal_state, float *dq, float *dk, float *dv,
                                    float *dg, float *dbeta, float *dinitial_state, int B, int T,
                                    int H, int dk_, int dv_, int num_seqs, kda_dtype dtype,
                                    void *stream) {
    t_msg[0] = 0;
    int N = 0;
    kda_status s = check_chunk_bwd_args("kda_chunk_bwd", q, k, v, g, beta, initial_state, cu_seqlens,
                                        dout, dfinal_state, dq, dk, dv, dg, dbeta, dinitial_state, B,
                                        T, H, dk_, dv_, num_seqs, dtype, &N);
    if (s != KDA_OK) return s;
    return chunk_bwd_run("kda_chunk_bwd", q, k, v, g, beta, initial_state, cu_seqlens, dout,
                         dfinal_state, dq, dk, dv, dg, dbeta, dinitial_state, B, T, H, N, nullptr,
                         (cudaStream_t)stream);
}

extern "C" long long kda_chunk_saved_bytes(int B, int T, int H, int num_seqs, int varlen) {
    if (B <= 0 || T < 0 || H <= 0 || B > 65535 || H > 65535 || (varlen && (B != 1 || num_seqs <= 0 ||
                                                                              num_seqs > 65535)))
        return -1;
    if ((long long)B * T > 0x7fffffffLL) return -1;
    return (long long)saved_layout(varlen ? num_seqs : B, B, T, H, varlen != 0).total;
}

extern "C" kda_status kda_chunk_fwd_save(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta,
                                         const float *initial_state, const int32_t *cu_seqlens,
                                         void *out, float *final_state, int B, int T, int H,
                                         int dk, int dv, int num_seqs, kda_dtype dtype, void *saved,
                                         long long saved_bytes, void *stream) {
    t_msg[0] = 0;
    int N = 0;
    kda_status s = kda::check_chunk_fwd_args("kda_chunk_fwd_save", q, k, v, g, beta, initial_state,
                                             cu_seqlens, out, final_state, B, T, H, dk, dv,
                                             num_seqs, dtype, &N);
    if (s != KDA_OK) return s;
    if (dtype != KDA_BF16 || dk != 128 || dv != 128)
        return fail(KDA_ERR_UNSUPPORTED,
                    "kda_chunk_fwd_save: only bf16 with dk = dv = 128 (got dtype %d, %d, %d)",
                    (int)dtype, dk, dv);
    const SavedLayout L = saved_layout(N, B, T, H, cu_seqlens != nullptr);
    if (!saved || ((uintptr_t)saved & 255u))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_save: saved must be 256-byte aligned");
    if (saved_bytes < (long long)L.total)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_save: saved holds %lld bytes, needs %zu",
                    saved_bytes, L.total);
    cudaStream_t st = (cudaStream_t)stream;
    const long long total_T = (long long)B * T;
    if (total_T == 0) {
        cudaError_t e = kda::bf16_prefill_no_tokens(initial_state, final_state, N, H, st);
        return e == cudaSuccess ? KDA_OK : cuda_fail(e, "kda_chunk_fwd_save empty input");
    }
    unsigned char *base = (unsigned char *)saved;
    int32_t *coff = (int32_t *)(base + L.plan);
    int32_t *order = cu_seqlens ? coff + N + 1 : nullptr;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int dvt = kda::bf16_prefill_dvt((long long)N * H, sms);
    int *err = kda::error_word();
    cudaError_t e = cudaSuccess;
    if (cu_seqlens) e = kda::launch_chunk_plan(cu_seqlens, N, (int)total_T, coff, st, order);
    if (e == cudaSuccess)
        e = kda::launch_chunk_prep(q, k, v, g, beta, cu_seqlens, coff, N, T, (int)total_T, H,
                                   (int)L.max_chunks, base + L.records, kda::Prologue{0, 1.f}, err, st);
    if (e == cudaSuccess)
        e = kda::launch_chunk_chain(base + L.records, cu_seqlens, coff, initial_state, final_state,
                                    out, N, T, (int)total_T, H, dvt, (int)L.max_chunks, err, st,
                                    base + L.s_img, base + L.v_img, order);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_save launch");
    return KDA_OK;
}

extern "C" kda_status kda_chunk_bwd_saved(const void *q, const void *k, const void *v,
                                          const float *g, const float *beta,
                                          const float *initial_state, const int32_t *cu_seqlens,
                                          const void *dout, const float *dfinal_state, float *dq,
                                          float *dk, float *dv, float *dg, float *dbeta,
                                          float *dinitial_state, int B, int T, int H, int dk_,
                                          int dv_, int num_seqs, kda_dtype dtype,
                                          const void *saved, long long saved_bytes, void *stream) {
    t_msg[0] = 0;
    int N = 0;
    kda_status s = check_chunk_bwd_args("kda_chunk_bwd_saved", q, k, v, g, beta, initial_state,
                                        cu_seqlens, dout, dfinal_state, dq, dk, dv, dg, dbeta,
                                        dinitial_state, B, T, H, dk_, dv_, num_seqs, dtype, &N);
    if (s != KDA_OK) return s;
    const SavedLayout L = saved_layout(N, B, T, H, cu_seqlens != nullptr);
    if (!saved || ((uintptr_t)saved & 255u))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_saved: saved must be 256-byte aligned");
    if (saved_bytes < (long long)L.total)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_bwd_saved: saved holds %lld bytes, needs %zu",
                    saved_bytes, L.total);
    return chunk_bwd_run("kda_chunk_bwd_saved", q, k, v, g, beta, initial_state, cu_seqlens, dout,
                         dfinal_state, dq, dk, dv, dg, dbeta, dinitial_state, B, T, H, N,
                         (const unsigned char *)saved, (cudaStream_t)stream);
}

extern "C" kda_status kda_recurrent_bwd(const void *q, const void *k, const void *v,
                                        const float *g, const float *beta,
                                        const float *initial_state, const void *dout,
                                        const float *dfinal_state, float *dq, float *dk,
                                        float *dv, float *dg, float *dbeta,
                                        float *dinitial_state, int B, int T, int H, int dk_,
                                        int dv_, kda_dtype dtype, void *stream) {
    t_msg[0] = 0;
    if (!q || !k || !v || !g || !beta || !dout || !dq || !dk || !dv || !dg || !dbeta)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_bwd: null pointer argument");
    if (B <= 0 || T <= 0 || H <= 0 || dk_ <= 0 || dv_ <= 0 || B > 65535 || H > 65535)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_bwd: bad sizes B=%d T=%d H=%d dk=%d dv=%d",
                    B, T, H, dk_, dv_);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_bwd: unknown dtype %d", (int)dtype);
    if (!((dk_ == 64 || dk_ == 128) && (dv_ == 64 || dv_ == 128)))
        return fail(KDA_ERR_UNSUPPORTED, "kda_recurrent_bwd: dk=%d dv=%d (supported: 64, 128)",
                    dk_, dv_);
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(dout) ||
        !aligned16(dq) || !aligned16(dk) || !aligned16(dv) || !aligned16(dg) ||
        !aligned16(initial_state) || !aligned16(dfinal_state) || !aligned16(dinitial_state))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_bwd: pointers must be 16-byte aligned");
    if (((uintptr_t)beta & 3u) || ((uintptr_t)dbeta & 3u))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_bwd: beta and dbeta must be 4-byte aligned");
    if ((long long)B * T * H > (1LL << 34))
        return fail(KDA_ERR_INVALID_ARG, "kda_recurrent_bwd: problem too large");
    cudaStream_t st = (cudaStream_t)stream;
    cudaMemPool_t pool;
    int sms = 148;
    cudaError_t e = get_pool(&pool, &sms);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_bwd memory pool");
    void *ws = nullptr;
    e = cudaMallocFromPoolAsync(&ws, kda::recurrent_bwd_workspace(B, T, H, dk_, dv_), pool, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_bwd workspace allocation");
    e = kda::launch_recurrent_bwd(q, k, v, g, beta, initial_state, dout, dfinal_state, dq, dk, dv,
                                  dg, dbeta, dinitial_state, ws, B, T, H, dk_, dv_,
                                  dtype == KDA_BF16, st);
    cudaError_t e2 = cudaFreeAsync(ws, st);
    if (e != cudaSuccess) return cuda_fail(e, "kda_recurrent_bwd launch");
    if (e2 != cudaSuccess) return cuda_fail(e2, "kda_recurrent_bwd workspace release");
    return KDA_OK;
}

extern "C" kda_status kda_state_affine(const float *M, const float *B, const float *S_in,
                                       float *S_out, int count, int dk, int dv, void *stream) {
    t_msg[0] = 0;
    if (!M || !S_in || !S_out)
        return fail(KDA_ERR_INVALID_ARG, "kda_state_affine: null pointer argument");
    if (count < 0 || count > 65535 || dk <= 0 || dk > 65535 || dv <= 0 || dv > 4096)
        return fail(KDA_ERR_INVALID_ARG, "kda_state_affine: bad sizes count=%d dk=%d dv=%d", count,
                    dk, dv);
    if (((uintptr_t)M | (uintptr_t)S_in | (uintptr_t)S_out | (uintptr_t)B) & 3u)
        return fail(KDA_ERR_INVALID_ARG, "kda_state_affine: pointers must be 4-byte aligned");
    const size_t sb = (size_t)count * dk * dv * sizeof(float), mb = (size_t)count * dk * dk * sizeof(float);
    auto overlap = [](const void *a, size_t na, const void *b, size_t nb) {
        return (const char *)a < (const char *)b + nb && (const char *)b < (const char *)a + na;
    };
    if (count > 0 && (overlap(S_out, sb, S_in, sb) || overlap(S_out, sb, M, mb)))
        return fail(KDA_ERR_INVALID_ARG, "kda_state_affine: S_out overlaps S_in or M");
    cudaError_t e = kda::launch_state_affine(M, B, S_in, S_out, count, dk, dv, (cudaStream_t)stream);
    if (e != cudaSuccess) return cuda_fail(e, "kda_state_affine launch");
    return KDA_OK;
}

// ---------------------------------------------------------------------------
// kda_chunk_fwd_host: host buffers, pipelined over token ranges.
namespace {

struct HostPipeStreams {
    cudaStream_t in = nullptr, out = nullptr;
};
std::mutex g_pipe_mu;
HostPipeStreams g_pipe[64];

cudaError_t pipe_streams(HostPipeStreams **ps) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_pipe_mu);
    HostPipeStreams &p = g_pipe[dev];
    if (!p.in && (e = cudaStreamCreateWithFlags(&p.in, cudaStreamNonBlocking)) != cudaSuccess) return e;
    if (!p.out && (e = cudaStreamCreateWithFlags(&p.out, cudaStreamNonBlocking)) != cudaSuccess) return e;
    *ps = &p;
    return cudaSuccess;
}

}  // namespace

extern "C" kda_status kda_chunk_fwd_host(const void *q, const void *k, const void *v,
                                         const float *g, const float *beta,
                                         const float *initial_state, const int32_t *cu_seqlens,
                                         void *out, float *final_state, int B, int T, int H,
                                         int dk, int dv, int num_seqs, kda_dtype dtype,
                                         int range_tokens, void *stream) {
    t_msg[0] = 0;
    if (!q || !k || !v || !g || !beta || !out)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: null pointer argument");
    if (B <= 0 || B > 65535 || T < 0 || H <= 0 || H > 65535 || dk <= 0 || dv <= 0 ||
        range_tokens < 0)
        return fail(KDA_ERR_INVALID_ARG,
                    "kda_chunk_fwd_host: bad sizes B=%d T=%d H=%d dk=%d dv=%d range_tokens=%d", B,
                    T, H, dk, dv, range_tokens);
    if (dtype != KDA_F32 && dtype != KDA_BF16)
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: unknown dtype %d", (int)dtype);
    if (!((dk == 64 || dk == 128) && (dv == 64 || dv == 128)))
        return fail(KDA_ERR_UNSUPPORTED, "kda_chunk_fwd_host: dk=%d dv=%d (supported: 64, 128)",
                    dk, dv);
    const long long total_T = (long long)B * T;
    if (total_T > 0x7fffffffLL || total_T * H > (1LL << 40))
        return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: problem too large (B*T=%lld)", total_T);
    // sequences on the packed token axis: dense [B, T] is B sequences of T
    int N = B;
    if (cu_seqlens) {
        if (B != 1)
            return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: varlen mode requires B == 1 (got %d)", B);
        if (num_seqs <= 0 || num_seqs > 65535)
            return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: num_seqs=%d out of [1, 65535]", num_seqs);
        N = num_seqs;
        // a host array: checked in full here
        if (cu_seqlens[0] != 0 || cu_seqlens[N] != T)
            return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: cu_seqlens must run from 0 to T=%d", T);
        for (int n = 0; n < N; ++n)
            if (cu_seqlens[n + 1] < cu_seqlens[n])
                return fail(KDA_ERR_INVALID_ARG, "kda_chunk_fwd_host: cu_seqlens decreases at %d", n);
    }
    auto seq_start = [&](int n) -> long long { return cu_seqlens ? cu_seqlens[n] : (long long)n * T; };
    cudaStream_t st = (cudaStream_t)stream;
    const size_t es = dtype == KDA_BF16 ? 2 : 4;
    const size_t one_state = (size_t)H * dk * dv * sizeof(float);
    const size_t state_bytes = (size_t)N * one_state;
    if (total_T == 0) {   // nothing to process: final = initial (or zeros)
        if (!final_state) return KDA_OK;
        cudaError_t e = initial_state
            ? cudaMemcpyAsync(final_state, initial_state, state_bytes, cudaMemcpyDefault, st)
            : cudaMemsetAsync(final_state, 0, state_bytes, st);
        if (e != cudaSuccess) {   // host memory cannot be memset by the device: zero it here
            if (initial_state) return cuda_fail(e, "kda_chunk_fwd_host empty input");
            cudaGetLastError();
            if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_host");
            memset(final_state, 0, state_bytes);
        }
        return KDA_OK;
    }
    // Ranges of the packed token axis that end at a sequence end or at a whole
    // number of chunks into a sequence, so every sequence keeps the chunk grid
    // of one call over it.  Range r covers tokens [cut[r], cut[r + 1]) and
    // the sequences first[r] .. last[r].
    int R = range_tokens > 0 ? range_tokens : 2048;
    R = (R + 63) / 64 * 64;
    auto seq_of = [&](long long p) -> int {   // the sequence holding token p
        if (!cu_seqlens) return (int)(p / T);
        int lo = 0, hi = N - 1;               // the last n with cu[n] <= p
        while (lo < hi) {
            const int mid = (lo + hi + 1) / 2;
            if (cu_seqlens[mid] <= p) lo = mid; else hi = mid - 1;
        }
        return lo;
    };
    std::vector<long long> cut{0};
    std::vector<int> first, last;
    for (long long t0 = 0; t0 < total_T;) {
        long long c = t0 + R;
        if (c >= total_T) {
            c = total_T;
        } else {   // back to the last chunk boundary of the sequence holding c
            const long long s = seq_start(seq_of(c));
            c = s + (c - s) / 64 * 64;    // > t0: t0 is itself such a boundary
        }
        first.push_back(seq_of(t0));
        last.push_back(seq_of(c - 1));
        cut.push_back(c);
        t0 = c;
    }
    const int nr = (int)first.size();
    long long max_tokens = 64;
    for (int r = 0; r < nr; ++r) max_tokens = std::max(max_tokens, cut[r + 1] - cut[r]);
    // per-token row bytes of each input / output (all heads)
    const size_t rq = (size_t)H * dk * es, rv = (size_t)H * dv * es, rg = (size_t)H * dk * 4,
                 rb = (size_t)H * 4, ro = (size_t)H * dv * es;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t Rt = (size_t)max_tokens;
    // one stage buffer: q k v g beta, each [range tokens, H, *]
    const size_t oq = 0, ok_ = al(Rt * rq), ov = ok_ + al(Rt * rq), og = ov + al(Rt * rv),
                 ob = og + al(Rt * rg);
    const size_t in_stage = ob + al(Rt * rb);
    const size_t out_stage = al(Rt * ro);
    // range-local offsets: nr arrays of (sequences + 1) int32
    std::vector<int32_t> local_cu;
    std::vector<size_t> cu_off(nr);
    for (int r = 0; r < nr; ++r) {
        cu_off[r] = local_cu.size();
        local_cu.push_back(0);
        for (int n = first[r]; n <= last[r]; ++n) {
            long long e_ = std::min(seq_start(n + 1), cut[r + 1]) - cut[r];
            local_cu.push_back((int32_t)e_);
        }
    }
    const size_t cu_bytes = al(local_cu.size() * sizeof(int32_t));
    const size_t total = 2 * in_stage + 2 * out_stage + al(state_bytes) + cu_bytes;

    HostPipeStreams *ps = nullptr;
    cudaMemPool_t pool;
    int sms = 148;
    cudaError_t e = pipe_streams(&ps);
    if (e == cudaSuccess) e = get_pool(&pool, &sms);
    if (e != cudaSuccess) return cuda_fail(e, "kda_chunk_fwd_host setup");
    void *buf = nullptr;
    if ((e = cudaMallocFromPoolAsync(&buf, total, pool, st)) != cudaSuccess)
        return cuda_fail(e, "kda_chunk_fwd_host device buffers");
    unsigned char *in_dev[2] = {(unsigned char *)buf, (unsigned char *)buf + in_stage};
    unsigned char *out_dev[2] = {in_dev[1] + in_stage, in_dev[1] + in_stage + out_stage};
    float *state_dev = (float *)(out_dev[1] + out_stage);
    int32_t *cu_dev = (int32_t *)((unsigned char *)state_dev + al(state_bytes));

    // events: start (buffers allocated, caller's prior work done), and per range
    // in_ready[r], done[r] (inputs of stage r % 2 free again), out_free[r]
    const int ne = 1 + 3 * nr;
    std::vector<cudaEvent_t> ev((size_t)ne);
    int made = 0;
    for (; made < ne; ++made)
        if ((e = cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming)) != cudaSuccess) break;
    kda_status status = KDA_OK;
    if (e != cudaSuccess) status = cuda_fail(e, "kda_chunk_fwd_host events");
    cudaEvent_t ev_start = ev[0];
    auto in_ready = [&](int r) { return ev[1 + 3 * r]; };
    auto done = [&](int r) { return ev[2 + 3 * r]; };
    auto out_free = [&](int r) { return ev[3 + 3 * r]; };
    auto chk = [&](cudaError_t x, const char *what) {
        if (status == KDA_OK && x != cudaSuccess) status = cuda_fail(x, what);
    };

    if (status == KDA_OK) {
        chk(cudaEventRecord(ev_start, st), "kda_chunk_fwd_host record");
        chk(cudaStreamWaitEvent(ps->in, ev_start, 0), "kda_chunk_fwd_host wait");
        chk(cudaStreamWaitEvent(ps->out, ev_start, 0), "kda_chunk_fwd_host wait");
        // every sequence's state lives in state_dev for the whole call
        chk(initial_state
                ? cudaMemcpyAsync(state_dev, initial_state, state_bytes, cudaMemcpyDefault, st)
                : cudaMemsetAsync(state_dev, 0, state_bytes, st),
            "kda_chunk_fwd_host initial state");
        chk(cudaMemcpyAsync(cu_dev, local_cu.data(), local_cu.size() * sizeof(int32_t),
                            cudaMemcpyHostToDevice, st),
            "kda_chunk_fwd_host range offsets");
    }
    for (int r = 0; r < nr && status == KDA_OK; ++r) {
        const long long t0 = cut[r];
        const int tr = (int)(cut[r + 1] - t0);
        const int b = r & 1;
        unsigned char *in = in_dev[b];
        // copy in (the stage's previous user, range r - 2, must be done)
        if (r >= 2) chk(cudaStreamWaitEvent(ps->in, done(r - 2), 0), "kda_chunk_fwd_host wait");
        const struct { const void *h; size_t off, row; } srcs[5] = {
            {q, oq, rq}, {k, ok_, rq}, {v, ov, rv}, {g, og, rg}, {beta, ob, rb}};
        for (const auto &c : srcs)
            chk(cudaMemcpyAsync(in + c.off, (const unsigned char *)c.h + (size_t)t0 * c.row,
                                (size_t)tr * c.row, cudaMemcpyDefault, ps->in),
                "kda_chunk_fwd_host copy in");
        chk(cudaEventRecord(in_ready(r), ps->in), "kda_chunk_fwd_host record");
        // compute on the caller's stream; the states of the range's sequences
        // are resumed and written back in place
        chk(cudaStreamWaitEvent(st, in_ready(r), 0), "kda_chunk_fwd_host wait");
        if (r >= 2) chk(cudaStreamWaitEvent(st, out_free(r - 2), 0), "kda_chunk_fwd_host wait");
        if (status != KDA_OK) break;
        float *sr = state_dev + (size_t)first[r] * (one_state / sizeof(float));
        const int nseq = last[r] - first[r] + 1;
        kda_status s2 = chunk_fwd_device(in + oq, in + ok_, in + ov, (const float *)(in + og),
                                         (const float *)(in + ob), sr, cu_dev + cu_off[r],
                                         out_dev[b], sr, 1, tr, H, dk, dv, nseq, dtype,
                                         kda::Prologue{0, 1.f}, st);
        if (s2 != KDA_OK) { status = s2; break; }
        chk(cudaEventRecord(done(r), st), "kda_chunk_fwd_host record");
        // copy out
        chk(cudaStreamWaitEvent(ps->out, done(r), 0), "kda_chunk_fwd_host wait");
        chk(cudaMemcpyAsync((unsigned char *)out + (size_t)t0 * ro, out_dev[b], (size_t)tr * ro,
                            cudaMemcpyDefault, ps->out),
            "kda_chunk_fwd_host copy out");
        chk(cudaEventRecord(out_free(r), ps->out), "kda_chunk_fwd_host record");
    }
    if (status == KDA_OK && final_state)
        chk(cudaMemcpyAsync(final_state, state_dev, state_bytes, cudaMemcpyDefault, st),
            "kda_chunk_fwd_host final state");
    // the caller's stream ends after every copy; buffers are released on it
    if (made == ne) {
        for (int r = 0; r < nr; ++r) {
            cudaStreamWaitEvent(st, in_ready(r), 0);
            cudaStreamWaitEvent(st, out_free(r), 0);
        }
    } else {
        cudaStreamSynchronize(ps->in);
        cudaStreamSynchronize(ps->out);
    }
    cudaError_t ef = cudaFreeAsync(buf, st);
    for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
    if (status == KDA_OK && ef != cudaSuccess) status = cuda_fail(ef, "kda_chunk_fwd_host release");
    return status;
}
