// prep_common.cuh -- helpers shared by the bf16 chunk prep (chunk_prep.cu)
// and the chunked backward (chunk_bwd.cu): the chunk locator, the blocked
// inverse T = (I + A)^-1 on a 64 x 64 fp32 tile, small conversions, the 3-D
// TMA load, and the tensor maps over [tokens, heads, 128] inputs.
#pragma once

#include <cudaTypedefs.h>

#include <mutex>

#include "chunk_ws.h"
#include "common.cuh"
#include "sm100.cuh"

namespace kda {
namespace prep {

constexpr int C = ws::C;
constexpr int D = ws::D;
constexpr int NT = 256;      // threads of a prep (and per-chunk backward) CTA

// 64 x 64 fp32 matrix, column groups of 4 XOR-swizzled by row
__device__ __forceinline__ int fsw(int i, int j) { return i * 64 + (j ^ ((i & 7) << 2)); }
// C(16x8) += X[r0:r0+16, kx0:kx0+K] Y[ky0:ky0+K, n0:n0+8], both in the fsw layout
template <int K>
__device__ __forceinline__ void tile_tf32(float (&c)[4], const float *X, int r0, int kx0,
                                          const float *Y, int ky0, int n0, int gid, int tig) {
#pragma unroll
    for (int ks = 0; ks < K; ks += 8) {
        const uint32_t a[4] = {to_tf32(X[fsw(r0 + gid, kx0 + ks + tig)]),
                               to_tf32(X[fsw(r0 + gid + 8, kx0 + ks + tig)]),
                               to_tf32(X[fsw(r0 + gid, kx0 + ks + tig + 4)]),
                               to_tf32(X[fsw(r0 + gid + 8, kx0 + ks + tig + 4)])};
        mma_tf32(c, a, to_tf32(Y[fsw(ky0 + ks + tig, n0 + gid)]),
                 to_tf32(Y[fsw(ky0 + ks + tig + 4, n0 + gid)]));
    }
}
__device__ __forceinline__ void store_tile(float *Mx, const float (&c)[4], int r0, int n0,
                                           int gid, int tig, float sgn) {
    Mx[fsw(r0 + gid, n0 + 2 * tig)] = sgn * c[0];
    Mx[fsw(r0 + gid, n0 + 2 * tig + 1)] = sgn * c[1];
    Mx[fsw(r0 + gid + 8, n0 + 2 * tig)] = sgn * c[2];
    Mx[fsw(r0 + gid + 8, n0 + 2 * tig + 1)] = sgn * c[3];
}

// Token range [t0, t0 + len) of global chunk `chunk` (dense: cps chunks per
// sequence of T tokens; varlen: coff[n] chunks before sequence n).
__device__ __forceinline__ void locate_chunk(int chunk, const int32_t *cu, const int32_t *coff,
                                             int N, int T, int total_T, int cps, long long &t0,
                                             int &len) {
    long long bos, eos;
    int cidx;
    if (cu) {
        int lo = 0, hi = N;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (coff[mid] <= chunk) lo = mid; else hi = mid;
        }
        bos = min(max(cu[lo], 0), total_T);
        eos = min(max(cu[lo + 1], 0), total_T);
        if (eos < bos) eos = bos;
        cidx = chunk - coff[lo];
    } else {
        const int seq = chunk / cps;
        cidx = chunk - seq * cps;
        bos = (long long)seq * T;
        eos = bos + T;
    }
    t0 = bos + (long long)C * cidx;
    len = (int)max(0LL, min((long long)C, eos - t0));
}

// form_T for the tensor-core prep: the diagonal 16x16 blocks of A come from a
// plain padded copy Ad[4][16][17] (row stride 17 floats: immediate offsets,
// no bank conflicts) and thread 0 first waits for its outstanding bulk
// stores to have read their shared-memory source (the caller reuses it).
// Zs may overlap Ad: Ad is dead after the diagonal step.
__device__ __forceinline__ void form_T_padded_diag(const float *Am, const float *Ad, float *Tm,
                                                   float *Zs, int tid) {
    const int lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    if (warp < 2) {
        const int Bk = 2 * warp + (lane >> 4), c = lane & 15, o = 16 * Bk;
        const float *ab = Ad + Bk * (16 * 17);
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float s = 0.f;
#pragma unroll
            for (int j = 0; j < i; ++j) s = fmaf(ab[i * 17 + j], x[j], s);
            x[i] = (i < c) ? 0.f : (i == c) ? 1.f : -s;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) Tm[fsw(o + i, o + c)] = x[i];
    } else {
        for (int e = tid - 64; e < 6 * 256; e += NT - 64) {
            const int blk = e >> 8, w = e & 255;
            const int Ib = blk < 3 ? 0 : blk < 5 ? 1 : 2;
            const int Jb = blk < 3 ? blk + 1 : blk < 5 ? blk - 1 : 3;
            Tm[fsw(16 * Ib + (w >> 4), 16 * Jb + (w & 15))] = 0.f;
        }
    }
    __syncthreads();
    if (warp < 4) {
        const int Ib = (warp >> 1) ? 3 : 1, Jb = Ib - 1, n0 = 16 * Jb + 8 * (warp & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<16>(c, Am, 16 * Ib, 16 * Jb, Tm, 16 * Jb, n0, gid, tig);
        store_tile(Zs, c, 16 * Ib, n0, gid, tig, 1.f);
    }
    __syncthreads();
    if (warp < 4) {
        const int Ib = (warp >> 1) ? 3 : 1, Jb = Ib - 1, n0 = 16 * Jb + 8 * (warp & 1);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<16>(c, Tm, 16 * Ib, 16 * Ib, Zs, 16 * Ib, n0, gid, tig);
        store_tile(Tm, c, 16 * Ib, n0, gid, tig, -1.f);
    }
    __syncthreads();
    {
        const int r0 = 32 + 16 * (warp >> 2), n0 = 8 * (warp & 3);
        float c[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<32>(c, Am, r0, 0, Tm, 0, n0, gid, tig);
        store_tile(Zs, c, r0, n0, gid, tig, 1.f);
        __syncthreads();
        float z[4] = {0.f, 0.f, 0.f, 0.f};
        tile_tf32<32>(z, Tm, r0, 32, Zs, 32, n0, gid, tig);
        store_tile(Tm, z, r0, n0, gid, tig, -1.f);
    }
    if (tid == 0) sm100::bulk_wait_read();
    __syncthreads();
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 bf16x2_to_float2(uint32_t x) {
    return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float2 v) { return pack_bf16(v.x, v.y); }
// 3-D tiled TMA load (no multicast) completing on an mbarrier
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, int x, int y, int z,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];\n"
        ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z),
          "r"(smem_u32(bar))
        : "memory");
}


}  // namespace prep

namespace prep {
// cuTensorMapEncodeTiled through the runtime's driver entry point (no link
// against the driver library)
static PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult res;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &res) == cudaSuccess &&
            res == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Tensor map over a [total_T, H, 128] tensor of `elem`-byte elements, boxes
// of {box_c channels, 1 head, 64 tokens}.
static cudaError_t make_token_map(CUtensorMap *m, const void *base, CUtensorMapDataType dt, int elem,
                                  int H, int total_T, int box_c, CUtensorMapSwizzle swz) {
    PFN_cuTensorMapEncodeTiled_v12000 fn = tensor_map_encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)total_T};
    const cuuint64_t strides[2] = {(cuuint64_t)D * elem, (cuuint64_t)D * elem * H};
    const cuuint32_t box[3] = {(cuuint32_t)box_c, 1, (cuuint32_t)C};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, dt, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace prep
}  // namespace kda
