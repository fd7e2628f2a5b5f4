// common.cuh -- small device helpers shared by the KDA kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Device error word: kernels that wait on barriers receive its address and
// set it (never trap) when a bounded wait runs out; kda_get_device_error()
// reads and clears it.  The word itself is defined in api.cu.
enum DeviceError : int {
    kErrNone = 0,
    kErrWaitTimeout = 1,     // an mbarrier wait exceeded its bound
    kErrBadOffsets = 2,      // cu_seqlens inconsistent (chunks beyond the records)
    kErrBadSlot = 3,         // a state-slot index outside [0, num_slots)
    kErrBwdRange = 4,        // chunked backward: a chunk's decay leaves e^{+-80} (chunk skipped)
};

// Input prologue (struct Prologue, kernels.h): q <- q_scale * (QK_L2NORM ?
// q / |q|_2 : q), k <- k / |k|_2 (QK_L2NORM; a zero row stays zero),
// beta <- sigmoid(beta) (BETA_SIGMOID).
constexpr int kProQkL2Norm = 1;
constexpr int kProBetaSigmoid = 2;
__device__ __forceinline__ float inv_norm(float sumsq) { return sumsq > 0.f ? rsqrtf(sumsq) : 0.f; }
__device__ __forceinline__ float sigmoid_f(float x) { return 1.f / (1.f + expf(-x)); }

__device__ __forceinline__ void set_device_error(int *word, int code) {
    if (word) atomicCAS(word, 0, code);
}

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Streaming 128-bit global load / store (evict-first: data touched once).
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

}  // namespace kda

namespace kda {

// ---------------------------------------------------------------------------
// Warp-level bf16 tensor-core helpers (m16n8k16, fp32 accumulate) and the
// shared-memory fragment loads that feed them.
//
// Fragment ownership (lane = 4*gid + tig):
//   A 16x16 (row-major): a0 (gid, 2tig..+1)  a1 (gid+8, 2tig..)  a2 (gid, 2tig+8..)
//                        a3 (gid+8, 2tig+8..)
//   B 16x8  (k x n):     b0 (k = 2tig..+1, n = gid)  b1 (k = 2tig+8.., n = gid)
//   C 16x8  (fp32):      c0,c1 (gid, 2tig..+1)       c2,c3 (gid+8, 2tig..+1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4],
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// Four 8x8 b16 matrices; lane i supplies the row address of matrix i/8, row i%8.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *row_ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row_ptr)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *row_ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(row_ptr)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// 16-byte asynchronous global -> shared copy (L2 only).
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)),
                 "l"(gmem_src));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

}  // namespace kda

namespace kda {
// m16n8k8 tf32 MMA with fp32 accumulate.  Fragments (lane = 4*gid + tig):
//   A 16x8: a0 (gid, tig)  a1 (gid+8, tig)  a2 (gid, tig+4)  a3 (gid+8, tig+4)
//   B 8x8:  b0 (k = tig, n = gid)  b1 (k = tig+4, n = gid)
//   C 16x8: as for the bf16 shape.
__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
}  // namespace kda
