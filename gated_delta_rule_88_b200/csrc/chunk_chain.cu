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
constexpr int PB = D + 8;
constexpr int PP = C + 8;

template <int DVT>
struct ChainSmem {
    static constexpr int PV = DVT + 8;
    __nv_bfloat16 AW[2][2 * C][PB];   // rows 0-63: W, rows 64-127: Qg
    __nv_bfloat16 KT[2][C][PB];       // Kt
    __nv_bfloat16 Pm[2][C][PP];       // P
    __nv_bfloat16 Ut[2][C][PV];       // U tile
    float eGC[2][D];
    __nv_bfloat16 Sb[D][PV];          // bf16 copy of the state tile
    __nv_bfloat16 Vn[C][PV];          // V_new (bf16)
};

template <int DVT>
__device__ __forceinline__ void load_record(ChainSmem<DVT> &sm, int buf, const unsigned char *rec,
                                            int n0, int tid)
{
    // [W; Qg]: 128 rows x 256 B
    for (int i = tid; i < 2 * C * (D / 8); i += NT) {
        const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
        const size_t off = (r < C ? ws::OFF_W : ws::OFF_QG) + ((size_t)(r & (C - 1)) * D + c8) * 2;
        cp_async16(&sm.AW[buf][r][c8], rec + off);
    }
    for (int i = tid; i < C * (D / 8); i += NT) {
        const int r = i / (D / 8), c8 = (i % (D / 8)) * 8;
        cp_async16(&sm.KT[buf][r][c8], rec + ws::OFF_KT + ((size_t)r * D + c8) * 2);
    }
    for (int i = tid; i < C * (C / 8); i += NT) {
        const int r = i / (C / 8), c8 = (i % (C / 8)) * 8;
        cp_async16(&sm.Pm[buf][r][c8], rec + ws::OFF_P + ((size_t)r * C + c8) * 2);
    }
    for (int i = tid; i < C * (DVT / 8); i += NT) {
        const int r = i / (DVT / 8), c8 = (i % (DVT / 8)) * 8;
        cp_async16(&sm.Ut[buf][r][c8], rec + ws::OFF_U + ((size_t)r * D + n0 + c8) * 2);
    }
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
    extern __shared__ __align__(16) unsigned char smem_raw[];
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
    const int a_row = (lane & 7) + 8 * ((lane >> 3) & 1), a_col = 8 * (lane >> 4);
    const int bt_k = (lane & 7) + 8 * ((lane >> 3) & 1), bt_n = 8 * (lane >> 4);
    const int at_k = (lane & 7) + 8 * (lane >> 4), at_m = 8 * ((lane >> 3) & 1);

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
            ldsm_x4(a, &sm.AW[buf][16 * warp + a_row][16 * ks + a_col]);
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
                const __nv_bfloat162 u0 = *reinterpret_cast<const __nv_bfloat162 *>(&sm.Ut[buf][r0][c]);
                const __nv_bfloat162 u1 = *reinterpret_cast<const __nv_bfloat162 *>(&sm.Ut[buf][r0 + 8][c]);
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
                ldsm_x4(a, &sm.Pm[buf][16 * I + a_row][16 * ks + a_col]);
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
                ldsm_x4_t(a, &sm.KT[buf][16 * ks + at_k][16 * warp + at_m]);
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

cudaError_t launch_chunk_chain(const unsigned char *wsp, const int32_t *cu, const int32_t *coff,
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
