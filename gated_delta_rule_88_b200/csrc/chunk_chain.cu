// chunk_chain.cu -- the sequential inter-chunk pass of the bf16 KDA prefill
// (dk = dv = 128, C = 64), warp-level bf16 tensor cores (m16n8k16).
//
// Kimi Linear paper notes (paper-notes-site), section 3: only the fixed-size
// state passes between chunks; the output is the inter-chunk part plus the
// intra-chunk part.  With the per-chunk record of chunk_ws.h, for each chunk
// in order and one 'DVT'-column tile of the state S (fp32, dk x DVT):
//     V_new = U - W S                      (the u_t of the recurrence)
//     O     = Qg S + P V_new
//     S    <- Diag(e^{G_C}) S + Kt^T V_new
// One CTA per (sequence, head, dv tile); chunks are walked in order while the
// next chunk's record streams into the other shared-memory buffer
// (cp.async double buffering).
//
// Warp roles (8 warps): every warp multiplies 16 rows of [W; Qg] (128 x 128)
// by S (bf16 copy in shared memory).  Warps 0-3 turn their rows into V_new;
// warps 4-7 keep Qg S and add P V_new.  Then every warp updates 16 channel
// rows of the fp32 state, which lives in its accumulator registers, and
// writes their bf16 copy for the next chunk.
#include "chunk_ws.h"
#include "common.cuh"
#include "kernels.h"

namespace kda {
namespace {

constexpr int C = ws::C;
constexpr int D = ws::D;
constexpr int NT = 256;

template <int DVT>
struct __align__(1024) ChainSmem {
    static constexpr int PV = DVT + 8;
    static constexpr int UT = DVT > 32 ? DVT / 32 : 1;   // U tiles of 32 columns
    unsigned char AW[2][32768];       // [W; Qg], K-major SW128 image (chunk_ws.h)
    unsigned char KTT[2][16384];      // Kt^T, K-major SW128 image
    unsigned char Pm[2][8192];        // P, K-major SW128 image
    unsigned char Ut[2][UT * 4096];   // U tile(s), plain [64][32]
    float eGC[2][D];
    __nv_bfloat16 Sb[D][PV];          // bf16 copy of the state tile
    __nv_bfloat16 Vn[C][PV];          // V_new (bf16)
};

// byte offset of 16-byte chunk j (0..7) of row r in a SW128 image
__device__ __forceinline__ int sw_chunk(int r, int j) { return r * 128 + ((j ^ (r & 7)) << 4); }

template <int DVT>
__device__ __forceinline__ void load_record(ChainSmem<DVT> &sm, int buf, const unsigned char *rec,
                                            int n0, int tid)
{
    constexpr int UT = ChainSmem<DVT>::UT;
    for (int i = tid; i < 32768 / 16; i += NT) cp_async16(&sm.AW[buf][i * 16], rec + ws::OFF_AW + i * 16);
    for (int i = tid; i < 16384 / 16; i += NT) cp_async16(&sm.KTT[buf][i * 16], rec + ws::OFF_KTT + i * 16);
    for (int i = tid; i < 8192 / 16; i += NT) cp_async16(&sm.Pm[buf][i * 16], rec + ws::OFF_P + i * 16);
    const unsigned char *u = rec + ws::OFF_U + (size_t)(n0 >> 5) * ws::U_TILE;
    for (int i = tid; i < UT * 4096 / 16; i += NT) cp_async16(&sm.Ut[buf][i * 16], u + i * 16);
    if (tid < D / 4) cp_async16(&sm.eGC[buf][tid * 4], rec + ws::OFF_EGC + tid * 16);
}

template <int DVT>
__global__ void __launch_bounds__(NT, 1)
chunk_chain_kernel(const unsigned char *__restrict__ wsp, const int32_t *__restrict__ cu,
                   const int32_t *__restrict__ coff, const float *__restrict__ s0,
                   float *__restrict__ sT, __nv_bfloat16 *__restrict__ out, int T, int total_T,
                   int H, int cps, int max_chunks, int *__restrict__ err)
{
    constexpr int NTN = DVT / 8;      // n-tiles of 8 columns
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    ChainSmem<DVT> &sm = *reinterpret_cast<ChainSmem<DVT> *>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int gid = lane >> 2, tig = lane & 3;
    const int n0 = blockIdx.x * DVT, h = blockIdx.y, seq = blockIdx.z;

    long long bos, eos;
    int c_begin;
    if (cu) {
        bos = min(max(cu[seq], 0), total_T);
        eos = min(max(cu[seq + 1], 0), total_T);
        if (eos < bos) eos = bos;
        c_begin = coff[seq];
    } else {
        bos = (long long)seq * T;
        eos = bos + T;
        c_begin = seq * cps;
    }
    int nchunks = (int)((eos - bos + C - 1) / C);
    if (c_begin < 0 || c_begin + nchunks > max_chunks) {
        // offsets inconsistent with the records the prep pass wrote (only
        // possible with invalid cu_seqlens): process nothing out of range
        if (tid == 0) set_device_error(err, kErrBadOffsets);
        nchunks = max(0, min(nchunks, max_chunks - max(c_begin, 0)));
        if (c_begin < 0) nchunks = 0;
    }

    // fp32 state rows (channels) 16*warp + gid (+8), columns 8*nt + 2*tig (+1)
    float S[NTN][4];
    const size_t sbase = ((size_t)seq * H + h) * (size_t)D * D;
    {
        const int r0 = 16 * warp + gid;
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) {
            const int c = n0 + 8 * nt + 2 * tig;
            if (s0) {
                const float2 x0 = *reinterpret_cast<const float2 *>(s0 + sbase + (size_t)r0 * D + c);
                const float2 x1 = *reinterpret_cast<const float2 *>(s0 + sbase + (size_t)(r0 + 8) * D + c);
                S[nt][0] = x0.x; S[nt][1] = x0.y; S[nt][2] = x1.x; S[nt][3] = x1.y;
            } else {
                S[nt][0] = S[nt][1] = S[nt][2] = S[nt][3] = 0.f;
            }
            *reinterpret_cast<uint32_t *>(&sm.Sb[r0][8 * nt + 2 * tig]) = pack_bf16(S[nt][0], S[nt][1]);
            *reinterpret_cast<uint32_t *>(&sm.Sb[r0 + 8][8 * nt + 2 * tig]) = pack_bf16(S[nt][2], S[nt][3]);
        }
    }
    const unsigned char *rec0 = wsp + ((size_t)c_begin * H + h) * ws::RECORD;
    const size_t rec_stride = (size_t)H * ws::RECORD;
    if (nchunks > 0) load_record<DVT>(sm, 0, rec0, n0, tid);
    cp_async_commit();

    // ldmatrix lane offsets
    const int a_row = (lane & 7) + 8 * ((lane >> 3) & 1);
    const int bt_k = (lane & 7) + 8 * ((lane >> 3) & 1), bt_n = 8 * (lane >> 4);

    for (int ci = 0; ci < nchunks; ++ci) {
        const int buf = ci & 1;
        cp_async_wait<0>();
        __syncthreads();
        if (ci + 1 < nchunks) load_record<DVT>(sm, buf ^ 1, rec0 + (size_t)(ci + 1) * rec_stride, n0, tid);
        cp_async_commit();
        const long long t0 = bos + (long long)C * ci;

        // [W; Qg] S : 16 rows per warp
        float acc[NTN][4];
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            uint32_t a[4];
            {
                const int r = 16 * warp + a_row, jj = 2 * ks + (lane >> 4);
                ldsm_x4(a, &sm.AW[buf][(jj >> 3) * 16384 + sw_chunk(r, jj & 7)]);
            }
#pragma unroll
            for (int np = 0; np < NTN / 2; ++np) {
                uint32_t b[4];
                ldsm_x4_t(b, &sm.Sb[16 * ks + bt_k][16 * np + bt_n]);
                mma_bf16(acc[2 * np], a, b[0], b[1]);
                mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
            }
        }
        if (warp < 4) {
            // V_new = U - W S
            const int r0 = 16 * warp + gid;
#pragma unroll
            for (int nt = 0; nt < NTN; ++nt) {
                const int c = 8 * nt + 2 * tig;
                const int lc = (n0 & 31) + c;   // column within the loaded U tile(s)
                const unsigned char *ut = &sm.Ut[buf][(lc >> 5) * 4096 + ((lc & 31) << 1)];
                const __nv_bfloat162 u0 = *reinterpret_cast<const __nv_bfloat162 *>(ut + r0 * 64);
                const __nv_bfloat162 u1 = *reinterpret_cast<const __nv_bfloat162 *>(ut + (r0 + 8) * 64);
                *reinterpret_cast<uint32_t *>(&sm.Vn[r0][c]) =
                    pack_bf16(__low2float(u0) - acc[nt][0], __high2float(u0) - acc[nt][1]);
                *reinterpret_cast<uint32_t *>(&sm.Vn[r0 + 8][c]) =
                    pack_bf16(__low2float(u1) - acc[nt][2], __high2float(u1) - acc[nt][3]);
            }
        }
        __syncthreads();
        if (warp >= 4) {
            // O = Qg S + P V_new (P is lower triangular: k-blocks <= row block)
            const int I = warp - 4;
            for (int ks = 0; ks <= I; ++ks) {
                uint32_t a[4];
                ldsm_x4(a, &sm.Pm[buf][sw_chunk(16 * I + a_row, 2 * ks + (lane >> 4))]);
#pragma unroll
                for (int np = 0; np < NTN / 2; ++np) {
                    uint32_t b[4];
                    ldsm_x4_t(b, &sm.Vn[16 * ks + bt_k][16 * np + bt_n]);
                    mma_bf16(acc[2 * np], a, b[0], b[1]);
                    mma_bf16(acc[2 * np + 1], a, b[2], b[3]);
                }
            }
            const int r0 = 16 * I + gid;
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
                const long long t = t0 + r0 + 8 * hh;
                if (t < eos) {
                    __nv_bfloat16 *orow = out + ((size_t)t * H + h) * D + n0;
#pragma unroll
                    for (int nt = 0; nt < NTN; ++nt)
                        *reinterpret_cast<uint32_t *>(orow + 8 * nt + 2 * tig) =
                            pack_bf16(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
                }
            }
        }
        // S <- Diag(e^{G_C}) S + Kt^T V_new  (rows 16*warp .. +15)
        {
            const float e0 = sm.eGC[buf][16 * warp + gid], e1 = sm.eGC[buf][16 * warp + gid + 8];
#pragma unroll
            for (int nt = 0; nt < NTN; ++nt) {
                S[nt][0] *= e0; S[nt][1] *= e0; S[nt][2] *= e1; S[nt][3] *= e1;
            }
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
                uint32_t a[4];
                ldsm_x4(a, &sm.KTT[buf][sw_chunk(16 * warp + a_row, 2 * ks + (lane >> 4))]);
#pragma unroll
                for (int np = 0; np < NTN / 2; ++np) {
                    uint32_t b[4];
                    ldsm_x4_t(b, &sm.Vn[16 * ks + bt_k][16 * np + bt_n]);
                    mma_bf16(S[2 * np], a, b[0], b[1]);
                    mma_bf16(S[2 * np + 1], a, b[2], b[3]);
                }
            }
            const int r0 = 16 * warp + gid;
#pragma unroll
            for (int nt = 0; nt < NTN; ++nt) {
                *reinterpret_cast<uint32_t *>(&sm.Sb[r0][8 * nt + 2 * tig]) = pack_bf16(S[nt][0], S[nt][1]);
                *reinterpret_cast<uint32_t *>(&sm.Sb[r0 + 8][8 * nt + 2 * tig]) = pack_bf16(S[nt][2], S[nt][3]);
            }
        }
    }
    cp_async_wait<0>();
    if (sT) {
        const int r0 = 16 * warp + gid;
#pragma unroll
        for (int nt = 0; nt < NTN; ++nt) {
            const int c = n0 + 8 * nt + 2 * tig;
            *reinterpret_cast<float2 *>(sT + sbase + (size_t)r0 * D + c) = make_float2(S[nt][0], S[nt][1]);
            *reinterpret_cast<float2 *>(sT + sbase + (size_t)(r0 + 8) * D + c) = make_float2(S[nt][2], S[nt][3]);
        }
    }
}

template <int DVT>
cudaError_t launch_chain_t(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
                           const float *s0, float *sT, void *out, int N, int T, int total_T,
                           int H, int max_chunks, int *err, cudaStream_t st)
{
    const size_t smem = sizeof(ChainSmem<DVT>);
    cudaError_t e = cudaFuncSetAttribute(chunk_chain_kernel<DVT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(D / DVT, H, N);
    chunk_chain_kernel<DVT><<<grid, NT, smem, st>>>(wsp, cu, coff, s0, sT, (__nv_bfloat16 *)out, T,
                                                    total_T, H, (T + C - 1) / C, max_chunks, err);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_chain_mma(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
                                   const float *s0, float *sT, void *out, int N, int T, int total_T,
                                   int H, int dvt, int max_chunks, int *err, cudaStream_t st)
{
    switch (dvt) {
        case 16: return launch_chain_t<16>(wsp, cu, coff, s0, sT, out, N, T, total_T, H, max_chunks, err, st);
        case 32: return launch_chain_t<32>(wsp, cu, coff, s0, sT, out, N, T, total_T, H, max_chunks, err, st);
        case 64: return launch_chain_t<64>(wsp, cu, coff, s0, sT, out, N, T, total_T, H, max_chunks, err, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace kda

#include <stdlib.h>
namespace kda {
cudaError_t launch_chunk_chain(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
                               const float *s0, float *sT, void *out, int N, int T, int total_T,
                               int H, int dvt, int max_chunks, int *err, cudaStream_t st)
{
    static const char *mode = getenv("KDA_CHAIN");
    if (mode && mode[0] == 'm')
        return launch_chunk_chain_mma(wsp, cu, coff, s0, sT, out, N, T, total_T, H, dvt, max_chunks, err, st);
    return launch_chunk_chain_tc(wsp, cu, coff, s0, sT, out, N, T, total_T, H, dvt, max_chunks, err, st);
}
}  // namespace kda
