// gated_norm.cu -- the output epilogue of the KDA layer: a gated RMSNorm.
//
// Kimi Linear paper notes (paper-notes-site), section 7: the layer does not
// return the KDA readout directly; it applies FusedRMSNormGated (an RMSNorm
// with a sigmoid output gate) before the output projection.  Per (token,
// head) row x of dv values, with gate row z and weight w [dv]:
//     y = x / sqrt(mean(x^2) + eps) * w * sigmoid(z)
// One warp per row; the row is read once and written once (HBM-bound:
// 3 * dv * sizeof(dtype) bytes per row).
#include "common.cuh"
#include "kernels.h"

namespace kda {
namespace {

template <typename T, int DV>
__global__ void __launch_bounds__(256)
gated_rmsnorm_kernel(const T *__restrict__ x, const T *__restrict__ z, const float *__restrict__ w,
                     float eps, T *__restrict__ y, long long rows)
{
    constexpr int PER = DV / 32;                        // values per lane
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    const size_t base = (size_t)row * DV + lane * PER;
    float xv[PER], zv[PER];
#pragma unroll
    for (int e = 0; e < PER; ++e) { xv[e] = to_f(x[base + e]); zv[e] = to_f(z[base + e]); }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) ss = fmaf(xv[e], xv[e], ss);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float r = rsqrtf(ss / (float)DV + eps);
#pragma unroll
    for (int e = 0; e < PER; ++e)
        y[base + e] = from_f<T>(xv[e] * r * w[lane * PER + e] * sigmoid_f(zv[e]));
}

template <typename T>
cudaError_t launch_t(const void *x, const void *z, const float *w, float eps, void *y,
                     long long rows, int dv, cudaStream_t st)
{
    const long long blocks = (rows + 7) / 8;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    if (dv == 128)
        gated_rmsnorm_kernel<T, 128><<<(unsigned)blocks, 256, 0, st>>>(
            (const T *)x, (const T *)z, w, eps, (T *)y, rows);
    else if (dv == 64)
        gated_rmsnorm_kernel<T, 64><<<(unsigned)blocks, 256, 0, st>>>(
            (const T *)x, (const T *)z, w, eps, (T *)y, rows);
    else
        return cudaErrorInvalidValue;
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_rmsnorm(const void *x, const void *z, const float *w, float eps, void *y,
                                 long long rows, int dv, bool bf16, cudaStream_t st)
{
    if (rows == 0) return cudaSuccess;
    return bf16 ? launch_t<__nv_bfloat16>(x, z, w, eps, y, rows, dv, st)
                : launch_t<float>(x, z, w, eps, y, rows, dv, st);
}

}  // namespace kda

// ---------------------------------------------------------------------------
// State affine map S_out = M S_in + B for `count` independent blocks (the
// composition step of a sequence split into segments: a segment's chunk map
// is S_end = M S_start + B).  Block (i, r) computes row r of S_out[i]; thread
// n owns column n: M[i][r][:] is a broadcast read, S_in[i][k][:] a coalesced
// row.  fp32 throughout.
namespace kda {
namespace {

__global__ void __launch_bounds__(128)
state_affine_kernel(const float *__restrict__ M, const float *__restrict__ B,
                    const float *__restrict__ S, float *__restrict__ out, int dk, int dv)
{
    const int i = blockIdx.x, r = blockIdx.y;
    const float *m = M + ((size_t)i * dk + r) * dk;
    const float *s = S + (size_t)i * dk * dv;
    for (int n = threadIdx.x; n < dv; n += blockDim.x) {
        float acc = B ? B[((size_t)i * dk + r) * dv + n] : 0.f;
        for (int k = 0; k < dk; ++k) acc = fmaf(m[k], s[(size_t)k * dv + n], acc);
        out[((size_t)i * dk + r) * dv + n] = acc;
    }
}

}  // namespace

cudaError_t launch_state_affine(const float *M, const float *B, const float *S, float *out,
                                int count, int dk, int dv, cudaStream_t st)
{
    if (count == 0) return cudaSuccess;
    dim3 grid(count, dk);
    state_affine_kernel<<<grid, 128, 0, st>>>(M, B, S, out, dk, dv);
    return cudaGetLastError();
}

}  // namespace kda
